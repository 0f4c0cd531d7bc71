"""Pins of the oracle's fixed-width b-bit variant (CPU).

The variant is the "4-bit and 2-bit QSGD" of the claim "QSVRG, non-convex and
multi-GPU bucketed training" and the 4/8-bit of the curated limitations of "QSGD
(Quantized Stochastic Gradient Descent) with Elias Coding" (AIMech curated entry).
The page gives no bit layout; the reading (s = 2^(b-1) - 1 levels, a b-bit code
(sign << (b-1)) | k per coordinate, packed MSB-first) is pinned by hand-derived words,
and the quantisation by the Elias path, which draws the same levels."""

import numpy as np
import pytest

import oracle as oracle_mod
from quantized_gradient_compression_b200 import workloads as W


def _unpack(codes: np.ndarray, n: int, b: int) -> np.ndarray:
    """Codes of n coordinates read back with numpy: bit j of the stream is bit
    31 - (j mod 32) of word j div 32."""
    bits = np.unpackbits(codes.astype(">u4").view(np.uint8))[: n * b].reshape(n, b)
    return (bits * (1 << np.arange(b - 1, -1, -1))).sum(axis=1).astype(np.int64)


@pytest.mark.parametrize("b,s", [(2, 1), (4, 7), (8, 127), (3, 0), (16, 0)])
def test_levels_per_width(oracle_lib, b, s):
    assert oracle_lib.bbit_levels(b) == s


# Hand-derived words: every t = |v_i| * s / ||v|| below is an integer, so p = 0 and no
# random word can change a level.
#  b=4, v = (0, -7, 0..): ||v|| = 7, s/||v|| = 1, k_1 = 7, sign 1 -> code 1111 at bits 4..7
#  b=4, v = (2, -3, 6, 0..): ||v|| = 7, k = (2, 3, 6) -> codes 0010 1011 0110
#  b=2, v = (0, -1, 0, 0): s = 1, ||v|| = 1, k_1 = 1, sign 1 -> code 11 at bits 2..3
#  b=8, v = (127, 0, 0, 0): s = 127 = ||v||, k_0 = 127 -> code 0111 1111
#  b=4, v = (0, 14, 0..): ||v|| = 14, s/||v|| = 0.5, k_1 = 7 -> code 0111; decodes to
#       fl(14/7) * 7 = 14 (a norm other than s, so the decode's scale is pinned too)
GOLDEN = [
    (4, [0, -7, 0, 0, 0, 0, 0, 0], 8, [0x0F000000], [7.0]),
    (4, [2, -3, 6, 0, 0, 0, 0, 0], 8, [0x2B600000], [7.0]),
    (2, [0, -1, 0, 0], 4, [0x30000000], [1.0]),
    (8, [127, 0, 0, 0], 4, [0x7F000000], [127.0]),
    (4, [0, 14, 0, 0, 0, 0, 0, 0], 8, [0x07000000], [14.0]),
    # two buckets of 4 (b = 4): (0, 0, 7, 0) and (0, -7, 0, 0) -> 0000 0000 0111 0000 | 0000 1111 ...
    (4, [0, 0, 7, 0, 0, -7, 0, 0], 4, [0x00700F00], [7.0, 7.0]),
]


@pytest.mark.parametrize("b,v,d,words,norms", GOLDEN)
def test_hand_derived_words(oracle_lib, b, v, d, words, norms):
    v = np.array(v, dtype=np.float32)
    for seed in (0, 1, 12345):
        codes, got_norms, st = oracle_lib.bbit_encode(v, d, b, seed)
        assert st == 0
        assert [int(w) for w in codes] == words
        assert got_norms.tolist() == norms
    out, st = oracle_lib.bbit_decode(got_norms, codes, v.size, d, b)
    assert st == 0 and np.array_equal(out, v)  # every level is exact here


@pytest.mark.parametrize("b", [2, 4, 8])
@pytest.mark.parametrize("n,d", [(1000, 128), (4099, 512), (777, 100), (50, 3), (1, 1)])
def test_same_levels_and_values_as_the_elias_path(oracle_lib, b, n, d):
    s = oracle_lib.bbit_levels(b)
    v = W.layered(n, n + d + b)
    levels, norms, st = oracle_lib.quantize(v, d, s, seed=7)
    codes, bnorms, bst = oracle_lib.bbit_encode(v, d, b, seed=7)
    assert st == bst == 0
    assert np.array_equal(norms.view(np.uint32), bnorms.view(np.uint32))
    code = _unpack(codes, n, b)
    k = code & s
    sign = code >> (b - 1)
    assert np.array_equal(k, np.abs(levels))
    assert np.array_equal(sign, ((levels < 0)).astype(np.int64))
    assert not np.any((k == 0) & (sign == 1))
    # decoded values bit for bit as the Elias stream decodes
    words, offsets, _, _ = oracle_lib.encode(v, d, s, seed=7)
    ref, _ = oracle_lib.decode(words, offsets, n, d, s)
    out, st = oracle_lib.bbit_decode(bnorms, codes, n, d, b)
    assert st == 0
    assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))


def test_code_array_size_and_padding(oracle_lib):
    for n, b in [(0, 4), (1, 2), (16, 2), (17, 2), (9, 4), (5, 8)]:
        assert oracle_lib.bbit_code_words(n, b) == (n * b + 31) // 32
    v = W.normal(9, 1)
    codes, _, _ = oracle_lib.bbit_encode(v, 9, 4, 3)
    assert codes.size == 2 and (int(codes[1]) & 0x0FFFFFFF) == 0  # bits past n*b are zero


@pytest.mark.parametrize("kind", ["sign_on_zero", "negative_norm", "nan_norm", "zero_norm_with_code",
                                  "underflowing_scale_with_code"])
def test_malformed_flagged(oracle_lib, kind):
    b, d = 4, 8
    norms = np.array([7.0], np.float32)
    codes = np.array([0x2B600000], np.uint32)
    if kind == "sign_on_zero":
        codes = np.array([0x2B680000], np.uint32)  # coordinate 3: sign 1, k 0
    elif kind == "negative_norm":
        norms = np.array([-7.0], np.float32)
    elif kind == "nan_norm":
        norms = np.array([np.nan], np.float32)
    elif kind == "zero_norm_with_code":
        norms = np.array([0.0], np.float32)
    else:
        norms = np.array([np.uint32(1).view(np.float32)], np.float32)  # 2^-149 / 7 = 0
    _, st = oracle_lib.bbit_decode(norms, codes, d, d, b)
    assert st & oracle_mod.ST_BAD_STREAM


def test_zero_and_nonfinite_buckets(oracle_lib):
    v = np.zeros(16, np.float32)
    v[8:] = W.normal(8, 2)
    v[12] = np.inf
    codes, norms, st = oracle_lib.bbit_encode(v, 8, 4, 0)
    assert st & oracle_mod.ST_NONFINITE
    assert norms.tolist() == [0.0, 0.0] and not codes.any()
    out, st = oracle_lib.bbit_decode(norms, codes, 16, 8, 4)
    assert st == 0 and not out.view(np.uint32).any()  # +0.0 everywhere


def test_decode_accumulate_is_sequential_sums(oracle_lib):
    n, d, b = 1000, 100, 2
    streams, qs = [], []
    for j in range(3):
        codes, norms, _ = oracle_lib.bbit_encode(W.normal(n, 40 + j), d, b, seed=j)
        streams.append((norms, codes))
        qs.append(oracle_lib.bbit_decode(norms, codes, n, d, b)[0])
    base = W.normal(n, 9) * np.float32(1e-2)
    base[::7] = np.float32(-0.0)
    out = base.copy()
    _, st = oracle_lib.bbit_decode_accumulate(streams, n, d, b, out)
    ref = base.copy()
    for q in qs:
        ref = (ref + q).astype(np.float32)
    assert st == 0 and np.array_equal(out.view(np.uint32), ref.view(np.uint32))


def test_rejects_other_widths(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.bbit_encode(np.ones(8, np.float32), 8, 3, 0)

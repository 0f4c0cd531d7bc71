"""Round trips, the size bound, decode-accumulate and malformed streams (oracle, CPU)."""

import itertools

import numpy as np
import pytest

import oracle as oracle_mod
from helpers import bits_to_words
from quantized_gradient_compression_b200 import workloads


def _vec(n, seed, kind="normal"):
    return workloads.GENERATORS[kind](n, seed)


@pytest.mark.parametrize("n,d,s", [(1, 1, 1), (7, 3, 2), (1000, 512, 16), (4099, 128, 4),
                                   (3000, 3000, 256), (2500, 1, 7), (777, 64, 1 << 22)])
def test_round_trip_levels(oracle_lib, n, d, s):
    v = _vec(n, n + d + s)
    levels, norms, st = oracle_lib.quantize(v, d, s, seed=11)
    words, offsets, enorms, st2 = oracle_lib.encode(v, d, s, seed=11)
    dl, dnorms, st3 = oracle_lib.decode_levels(words, offsets, n, d, s)
    assert st == st2 == st3 == 0
    assert np.array_equal(levels, dl)
    assert np.array_equal(norms.view(np.uint32), dnorms.view(np.uint32))
    assert np.array_equal(norms.view(np.uint32), enorms.view(np.uint32))
    assert np.all(np.abs(levels) <= s)


def test_decoded_values_follow_levels(oracle_lib):
    n, d, s = 5000, 512, 16
    v = _vec(n, 3, "layered")
    words, offsets, norms, _ = oracle_lib.encode(v, d, s, seed=5)
    out, st = oracle_lib.decode(words, offsets, n, d, s)
    levels, _, _ = oracle_lib.decode_levels(words, offsets, n, d, s)
    assert st == 0
    # support and signs agree with the levels; magnitudes are |k| * norm/s
    assert np.array_equal(out != 0, levels != 0)
    assert np.array_equal(np.signbit(out[levels != 0]), levels[levels != 0] < 0)
    for b in range((n + d - 1) // d):
        seg = slice(b * d, min(n, (b + 1) * d))
        scale = np.float32(norms[b]) / np.float32(s)
        expect = np.abs(levels[seg]).astype(np.float32) * scale
        assert np.allclose(np.abs(out[seg]), expect, rtol=0, atol=0)


def test_same_seed_same_stream_other_seed_differs(oracle_lib):
    v = _vec(4096, 1)
    a = oracle_lib.encode(v, 512, 8, seed=1)
    b = oracle_lib.encode(v, 512, 8, seed=1)
    c = oracle_lib.encode(v, 512, 8, seed=2)
    assert np.array_equal(a[0], b[0])
    assert not np.array_equal(a[0], c[0])


def test_partition_invariance_of_randomness(oracle_lib):
    # the random word depends on the global index only: the levels of a bucket
    # do not depend on which other buckets exist
    v = _vec(2048, 9)
    full, _, _ = oracle_lib.quantize(v, 512, 16, seed=3)
    lib = oracle_lib.lib
    import ctypes
    st = ctypes.c_uint32(0)
    part = np.zeros(512, dtype=np.int32)
    vb = np.ascontiguousarray(v[1024:1536])
    lib.qo_quantize_bucket(vb.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), 512, 1024, 16, 3,
                           None, part.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                           ctypes.byref(st))
    assert np.array_equal(part, full[1024:1536])


def test_size_bound_brute_force(oracle_lib):
    # every support pattern of a bucket of m <= 12 coordinates, every level = s:
    # the record bits never exceed m * (2 + |omega(s)|)
    for s in [1, 2, 3, 4, 16, 255, 256, 1 << 22]:
        ws = oracle_lib.omega_len(s)
        for m in range(1, 13):
            worst = 0
            for mask in range(1, 1 << m):
                prev, bits = -1, 0
                for i in range(m):
                    if mask >> i & 1:
                        bits += oracle_lib.omega_len(i - prev) + 1 + ws
                        prev = i
                worst = max(worst, bits)
            assert worst + 32 <= oracle_lib.bucket_bit_bound(m, s)
            # the all-non-zero pattern with k = s meets the bound exactly
            assert worst + 32 == oracle_lib.bucket_bit_bound(m, s)


def test_gap_cost_bound(oracle_lib):
    for s in [1, 16, 256, 1 << 22]:
        ws = oracle_lib.omega_len(s)
        for g in list(range(1, 5000)) + [1 << 16, (1 << 20) + 3, 1 << 31]:
            assert oracle_lib.omega_len(g) + 1 + ws <= g * (2 + ws)


def test_capacity_covers_dense_worst_case(oracle_lib):
    # equal magnitudes: every coordinate is on the support
    n, d, s = 1000, 100, 256
    v = np.ones(n, dtype=np.float32)
    v[::3] = -1
    words, offsets, _, st = oracle_lib.encode(v, d, s, seed=0)
    assert st == 0
    assert int(offsets[-1]) <= 32 * oracle_lib.capacity_words(n, d, s)


def test_empty_vector(oracle_lib):
    words, offsets, norms, st = oracle_lib.encode(np.zeros(0, np.float32), 512, 4, seed=0)
    assert offsets.tolist() == [0] and words.size == 0 and st == 0
    out, st = oracle_lib.decode(words, offsets, 0, 512, 4)
    assert out.size == 0 and st == 0


def test_decode_accumulate_hand_values(oracle_lib):
    # (n, d, s) = (2, 2, 5).  Stream a: case A of the golden file, decodes to (3, 4).
    # Stream b: norm 2, one record at index 1: gap 2 = "100", sign 1, k = 1 = "0";
    # it decodes to (0, -fl(2/5)).
    a = bits_to_words("01000000101000000000000000000000" + "00110" + "00101000")
    b = bits_to_words("01000000000000000000000000000000" + "100" + "1" + "0")
    oa = np.array([0, 45], dtype=np.uint64)
    ob = np.array([0, 37], dtype=np.uint64)
    out_a, st = oracle_lib.decode(a, oa, 2, 2, 5)
    out_b, st2 = oracle_lib.decode(b, ob, 2, 2, 5)
    assert st == 0 and st2 == 0
    assert out_a.tolist() == [3.0, 4.0]
    assert out_b.view(np.uint32).tolist() == [0, int(np.float32(-0.4).view(np.uint32))]
    out = np.array([0.5, -0.0], dtype=np.float32)
    res, st3 = oracle_lib.decode_accumulate([(a, oa), (b, ob)], 2, 2, 5, out)
    assert st3 == 0
    f = np.float32
    expect = np.array([f(f(f(0.5) + f(3)) + f(0)), f(f(f(-0.0) + f(4)) + f(-0.4))], np.float32)
    assert res.view(np.uint32).tolist() == expect.view(np.uint32).tolist()


def test_underflowing_scale_with_records_is_flagged(oracle_lib):
    # norm = 2^-149 (bit pattern 1) and s = 8: fl(norm / s) = 0, and s / norm overflows,
    # so no encoder sends records under this norm.  One record gap 1, sign 0, k 1 = "000".
    s = 8
    tiny = bits_to_words("0" * 31 + "1" + "000")
    off = np.array([0, 35], dtype=np.uint64)
    out, st = oracle_lib.decode(tiny, off, 1, 1, s)
    assert st & oracle_mod.ST_BAD_STREAM
    assert np.float32(np.uint32(1).view(np.float32)) / np.float32(s) == 0
    # the same norm with no record is a valid (all-zero) bucket
    out, st = oracle_lib.decode(bits_to_words("0" * 31 + "1"), np.array([0, 32], np.uint64), 1, 1, s)
    assert st == 0 and out.view(np.uint32).tolist() == [0]
    # the smallest normal norm 2^-126 keeps a non-zero scale: the record decodes
    normal = bits_to_words("00000000100000000000000000000000" + "000")
    out, st = oracle_lib.decode(normal, off, 1, 1, s)
    assert st == 0 and out[0] == np.float32(2.0 ** -126) / np.float32(s) and out[0] > 0


def test_decode_accumulate_negative_zero_becomes_positive(oracle_lib):
    # -0.0 + (+0.0) = +0.0: a coordinate off every support turns -0 into +0
    z = bits_to_words("0" * 32)
    oz = np.array([0, 32], dtype=np.uint64)
    out = np.array([-0.0, -0.0], dtype=np.float32)
    res, st = oracle_lib.decode_accumulate([(z, oz)], 2, 2, 3, out)
    assert st == 0 and not np.signbit(res).any()


def test_decode_accumulate_matches_sequential_sums(oracle_lib):
    n, d, s, K = 3000, 512, 4, 3
    streams = []
    for j in range(K):
        v = _vec(n, 100 + j, "small_normal")
        w, o, _, _ = oracle_lib.encode(v, d, s, seed=j)
        streams.append((w, o))
    base = _vec(n, 77)
    out = base.copy()
    oracle_lib.decode_accumulate(streams, n, d, s, out)
    ref = base.copy()
    for w, o in streams:
        q, _ = oracle_lib.decode(w, o, n, d, s)
        ref = (ref + q).astype(np.float32)
    assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))


def _good_stream(oracle_lib):
    v = _vec(1024, 4)
    return oracle_lib.encode(v, 256, 4, seed=1)


@pytest.mark.parametrize("kind", ["truncate", "reverse_offsets", "short_bucket", "big_level",
                                  "bad_norm", "index_past_end"])
def test_malformed_streams_flagged(oracle_lib, kind):
    words, offsets, norms, _ = _good_stream(oracle_lib)
    words = words.copy()
    offsets = offsets.copy()
    n, d, s = 1024, 256, 4
    if kind == "truncate":
        offsets[2] -= 3
    elif kind == "reverse_offsets":
        offsets[1], offsets[2] = offsets[2], offsets[1]
    elif kind == "short_bucket":
        offsets[1] = offsets[0] + 20
    elif kind == "big_level":
        # a bucket whose only record is gap 1, sign 0, k = 5 > s (omega(5) = 101010)
        words = bits_to_words("01000000000000000000000000000000" + "0" + "0" + "101010")
        offsets = np.array([0, 40, 40, 40, 40], dtype=np.uint64)
    elif kind == "bad_norm":
        words = bits_to_words("11111111110000000000000000000000")  # a NaN norm
        offsets = np.array([0, 32, 32, 32, 32], dtype=np.uint64)
    elif kind == "index_past_end":
        # gap 300 > bucket length 256: omega(300) = 10 1000 100101100 0
        words = bits_to_words("01000000000000000000000000000000" + "10" + "1000" +
                              "100101100" + "0" + "0" + "0")
        offsets = np.array([0, 32 + 16 + 2, 0, 0, 0], dtype=np.uint64)
    _, st = oracle_lib.decode(words, offsets, n, d, s)
    assert st & oracle_mod.ST_BAD_STREAM


def test_range_status_for_tiny_norm(oracle_lib):
    v = np.array([1e-38, 0, 0, 0], dtype=np.float32)
    words, offsets, norms, st = oracle_lib.encode(v, 4, 1 << 22, seed=0)
    assert st & oracle_mod.ST_RANGE
    assert offsets.tolist() == [0, 32] and int(words[0]) == 0


@pytest.mark.parametrize("n,d,s", [(10_007, 100, 16), (4_096, 512, 1), (3_000, 7, 300)])
def test_encode_range_is_a_slice_of_the_whole_stream(oracle_lib, n, d, s):
    """encode_range(b0, b1) keeps every coordinate's global index (its Philox word):
    its stream is bits [offsets[b0], offsets[b1]) of the whole-vector stream, its
    offsets are the whole offsets shifted, and the slices tile the whole stream."""
    from gpu_common import extract_bits
    from quantized_gradient_compression_b200 import workloads as W

    v = W.layered(n, n % 13)
    words, offsets, norms, st = oracle_lib.encode(v, d, s, 21)
    nb = offsets.size - 1
    cuts = [0, 1, nb // 3, nb // 3 + 1, nb - 1, nb]
    for b0, b1 in zip(cuts[:-1], cuts[1:]):
        rw, ro, rn, rst = oracle_lib.encode_range(v, d, s, 21, b0, b1)
        begin, end = int(offsets[b0]), int(offsets[b1])
        assert np.array_equal(ro, offsets[b0:b1 + 1] - offsets[b0])
        assert np.array_equal(rn.view(np.uint32), norms[b0:b1].view(np.uint32))
        assert np.array_equal(rw, extract_bits(words, begin, end))
    # the GPU-norm form: with norms_in, the same slice as encode(norms_in=...)
    alt = norms * np.float32(1.0000001)
    aw, ao, _, _ = oracle_lib.encode(v, d, s, 21, norms_in=alt)
    rw, ro, _, _ = oracle_lib.encode_range(v, d, s, 21, 1, nb, norms_in=alt[1:])
    assert np.array_equal(rw, extract_bits(aw, int(ao[1]), int(ao[nb])))

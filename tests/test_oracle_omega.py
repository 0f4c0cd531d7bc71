"""Pins of the oracle's Elias omega code (Elias 1975, the recursive code)."""

import numpy as np
import pytest

from helpers import load_omega_codewords


@pytest.mark.parametrize("N,code", load_omega_codewords())
def test_textbook_codewords(oracle_lib, N, code):
    assert oracle_lib.omega_bits(N) == code
    assert oracle_lib.omega_len(N) == len(code)


def test_textbook_lengths(oracle_lib):
    # lengths worked out by hand from the omega construction (Elias 1975), e.g.
    # 16 -> 10 100 10000 0 (11 bits), 512 -> 11 1001 1000000000 0 (17 bits)
    expect = {1: 1, 2: 3, 3: 3, 4: 6, 8: 7, 16: 11, 256: 16, 512: 17, 8192: 21, 1 << 20: 32}
    for N, ln in expect.items():
        assert oracle_lib.omega_len(N) == ln


def test_brute_force_round_trip_1_to_2_pow_20(oracle_lib):
    """Every integer 1..2^20 encoded back to back in one stream decodes back."""
    values = np.arange(1, (1 << 20) + 1, dtype=np.uint64)
    words, nbits = oracle_lib.omega_put_many(values)
    decoded, pos = oracle_lib.omega_get_many(words, len(values), nbits)
    assert pos == nbits
    assert np.array_equal(np.asarray(decoded, dtype=np.uint64), values)
    total = sum(oracle_lib.omega_len(int(x)) for x in values)
    assert total == nbits


def test_length_is_log_plus_loglog(oracle_lib):
    # |omega(N)| = log2 N + O(log log N): for N >= 2 the code is binary(N) plus
    # the code of bitlength(N)-1 without its final 0, plus the final 0.
    for N in [2, 3, 5, 9, 100, 1000, 65535, 65536, 1 << 30, (1 << 40) + 7]:
        b = N.bit_length()
        assert oracle_lib.omega_len(N) == b + oracle_lib.omega_len(b - 1)


def test_monotone_lengths(oracle_lib):
    prev = 0
    for N in range(1, 5000):
        ln = oracle_lib.omega_len(N)
        assert ln >= prev
        prev = ln


def test_prefix_free_small(oracle_lib):
    codes = [oracle_lib.omega_bits(N) for N in range(1, 2049)]
    seen = set(codes)
    assert len(seen) == len(codes)
    for c in codes:
        for cut in range(1, len(c)):
            assert c[:cut] not in seen

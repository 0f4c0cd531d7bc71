"""Pins of the oracle's random source (Philox4x32-10, Salmon et al. SC'11)."""

import numpy as np
import pytest

from helpers import load_kat


@pytest.mark.parametrize("ctr,key,expect", load_kat())
def test_philox_known_answers(oracle_lib, ctr, key, expect):
    out = oracle_lib.philox(ctr, key)
    assert [int(x) for x in out] == expect


def test_random_word_uses_block_of_four(oracle_lib):
    # counter 0, key 0 is the first known-answer vector: coordinates 0..3 of
    # seed 0 take its four words in order.
    (ctr, key, expect) = load_kat()[0]
    assert [oracle_lib.random_word(0, i) for i in range(4)] == expect


def test_random_word_counter_and_key_layout(oracle_lib):
    # index i uses counter (lo32(i/4), hi32(i/4), 0, 0) and key (lo32(seed), hi32(seed))
    seed = 0x0123456789ABCDEF
    for i in [0, 5, 4 * 0x1_0000_0003 + 2]:
        j = i // 4
        out = oracle_lib.philox([j & 0xFFFFFFFF, j >> 32, 0, 0],
                                [seed & 0xFFFFFFFF, seed >> 32])
        assert oracle_lib.random_word(seed, i) == int(out[i % 4])


def test_uniform_grid_chi_square(oracle_lib):
    # u = floor(r/2^9)/2^23 must be uniform: chi-square over 64 cells of 2^16 draws.
    n = 1 << 16
    lib = oracle_lib.lib
    r = np.array([lib.qo_random_word(7, i) for i in range(n)], dtype=np.uint64)
    u = (r >> 9).astype(np.float64) / float(1 << 23)
    counts, _ = np.histogram(u, bins=64, range=(0.0, 1.0))
    expected = n / 64
    chi2 = float(((counts - expected) ** 2 / expected).sum())
    # 63 degrees of freedom: mean 63, sd ~11.2; 63 + 6 sd ~ 130
    assert chi2 < 130, chi2
    assert u.min() >= 0.0 and u.max() < 1.0

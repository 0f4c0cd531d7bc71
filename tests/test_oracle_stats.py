"""The page's distributional claims checked on the oracle (seed sweeps)."""

import numpy as np
import pytest

from quantized_gradient_compression_b200 import workloads
import stats_common as sc


@pytest.fixture(scope="module")
def sweep_c1():
    # the single-bucket vector, s = sqrt(n) = 256, seeds 0..9999
    v = workloads.C1.generate()
    return v, sc.sweep(v, 256, range(10_000))


def test_unbiased_10k_seeds(sweep_c1):
    v, sums = sweep_c1
    assert sums.count == 10_000
    sc.check_unbiased(v, 256, sums)


def test_variance_identity_and_bound(sweep_c1):
    v, sums = sweep_c1
    measured, closed, bound = sc.check_variance(v, 256, sums)
    # at s = sqrt(n) the blow-up min(n/s^2, sqrt(n)/s) is 1 (second moment <= 2x)
    assert bound == pytest.approx(float(np.sum(v.astype(np.float64) ** 2)))


def test_support_expectation(sweep_c1):
    v, sums = sweep_c1
    sc.check_support(v, 256, sums)


def test_support_bound_where_it_bites():
    # s = 16, n = 65536: s^2 + s sqrt(n) = 4352 < n, so the bound is not vacuous
    v = workloads.C1.generate()
    sums = sc.sweep(v, 16, range(1000))
    mean, expect, bound = sc.check_support(v, 16, sums)
    assert bound == 4352 and mean < bound
    sc.check_unbiased(v, 16, sums, max_beyond_4se=10)
    sc.check_variance(v, 16, sums)


def test_bits_at_s_sqrt_n_within_2_818n_plus_32(oracle_lib):
    # claim "Elias coding communication complexity tradeoff": at s = sqrt(n) the
    # expected stream is at most 2.818 n + 32 bits
    v = workloads.C1.generate()
    n = v.size
    bits = []
    for seed in range(200):
        _, offsets, _, st = oracle_lib.encode(v, n, 256, seed)
        assert st == 0
        bits.append(int(offsets[-1]))
    bits = np.asarray(bits, dtype=np.float64)
    assert bits.mean() + 4 * bits.std(ddof=1) / np.sqrt(bits.size) <= 2.818 * n + 32


def test_printed_general_bound_at_large_s(oracle_lib):
    # The same claim prints a general form (3/2 + 1/2 log2(2(s^2+n)/s)) s (s + sqrt n) + F.
    # Measured with the omega code it holds for s >= 16 but is BELOW the coded size
    # for s <= 8 (s = 1: ~3100 bits against 2602), so the printed expression is read
    # as garbled there; only the explicit 2.818 n + 32 statement is a hard pin.
    v = workloads.C1.generate()
    n = v.size
    for s in [16, 64, 256]:
        _, offsets, _, _ = oracle_lib.encode(v, n, s, 1)
        bound = (1.5 + 0.5 * np.log2(2 * (s * s + n) / s)) * s * (s + np.sqrt(n)) + 32
        assert int(offsets[-1]) <= bound
    _, offsets, _, _ = oracle_lib.encode(v, n, 1, 1)
    assert int(offsets[-1]) > (1.5 + 0.5 * np.log2(2 * (1 + n))) * (1 + np.sqrt(n)) + 32

"""Pins of the oracle's max-norm (QSGDinf) scale (CPU).

The NUQSGD abstract names QSGDinf as the authors' practical heuristic of QSGD; the
page gives no formula, and the name gives the norm: each bucket is scaled by
||v||_inf instead of ||v||_2, with the same quantiser and coding.  The max is exact,
so the oracle's value is fixed by numpy's; the quantiser with any scale >= max|v_i|
stays unbiased, checked over seeds."""

import numpy as np
import pytest

import oracle as oracle_mod
from quantized_gradient_compression_b200 import workloads as W


@pytest.mark.parametrize("kind,n", [("normal", 1000), ("layered", 4099), ("heavy_tailed_sparse", 777)])
def test_maxnorm_is_numpy_max_abs(oracle_lib, kind, n):
    v = W.GENERATORS[kind](n, n)
    for d in (1, 7, 128, n):
        got = oracle_lib.maxnorms(v, d)
        nb = (n + d - 1) // d
        ref = np.array([np.max(np.abs(v[b * d:(b + 1) * d])) for b in range(nb)], np.float32)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_maxnorm_special_values(oracle_lib):
    assert oracle_lib.bucket_maxnorm(np.zeros(5, np.float32)) == 0
    assert oracle_lib.bucket_maxnorm(np.array([1, -np.inf, 2], np.float32)) == np.inf
    assert np.isnan(oracle_lib.bucket_maxnorm(np.array([1, np.nan, np.inf], np.float32)))
    assert oracle_lib.bucket_maxnorm(np.array([-0.0, -3.5, 2], np.float32)) == 3.5


def test_maxnorm_scale_reaches_level_s_and_flags(oracle_lib):
    # the largest |v_i| of a bucket has t = fl(max * fl(s / max)); for this vector that
    # product rounds to s itself, so its level is s whatever the random word
    v = W.normal(512, 3)
    mx = oracle_lib.maxnorms(v, 512)
    assert np.float32(mx[0]) * np.float32(np.float32(16) / mx[0]) == np.float32(16)
    for seed in range(5):
        levels, norms, st = oracle_lib.quantize(v, 512, 16, seed, norms_in=mx)
        assert st == 0 and np.abs(levels[np.argmax(np.abs(v))]) == 16
    bad = v.copy()
    bad[3] = np.nan
    _, _, st = oracle_lib.quantize(bad, 512, 16, 0, norms_in=oracle_lib.maxnorms(bad, 512))
    assert st & oracle_mod.ST_NONFINITE


def test_maxnorm_quantiser_is_unbiased(oracle_lib):
    """E[k_i] = t_i = |v_i| * fl(s / ||v||_inf): mean level within 4 standard errors
    per coordinate (a handful of 4-SE excursions allowed), the near-deterministic
    coordinates summed together, over 2000 seeds."""
    v = W.normal(4096, 1)
    s = 8
    mx = oracle_lib.maxnorms(v, v.size)
    N = 2000
    k1 = np.zeros(v.size)
    for seed in range(N):
        levels, norms, _ = oracle_lib.quantize(v, v.size, s, seed, norms_in=mx)
        assert norms[0] == mx[0]
        k1 += np.abs(levels)
    sinv = np.float32(np.float32(s) / mx[0])
    t = (np.abs(v) * sinv).astype(np.float64)
    p = t - np.floor(t)
    var = p * (1 - p)
    mean_k = k1 / N
    live = var * N >= 10.0
    z = (mean_k[live] - t[live]) / np.sqrt(var[live] / N)
    assert np.count_nonzero(np.abs(z) > 4) <= 10 and np.max(np.abs(z)) < 6.5
    exact = p == 0.0
    assert np.all(mean_k[exact] == t[exact])
    few = ~live & ~exact
    dev = float(np.sum((mean_k[few] - t[few]) * N))
    assert abs(dev) <= 4 * np.sqrt(float(np.sum(var[few] * N))) + 1.0

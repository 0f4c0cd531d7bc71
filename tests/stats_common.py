"""Seed sweeps for the statistical checks of the quantiser's claims.

The expectations come from the real-number formulas of the definition paragraph
and the claim "unbiased stochastic quantization, variance and sparsity bounds" of
the page "QSGD (Quantized Stochastic Gradient Descent) with Elias Coding":
E[Q_s(v)] = v, E||Q_s(v) - v||^2 = (||v||^2/s^2) sum p_i (1 - p_i)
<= min(n/s^2, sqrt(n)/s) ||v||^2, E||Q_s(v)||_0 <= s^2 + s sqrt(n).
They are evaluated in float64 from v alone, never from the implementation.
"""

import multiprocessing as mp

import numpy as np


def exact_moments(v: np.ndarray, s: int):
    v64 = v.astype(np.float64)
    norm = np.sqrt(np.sum(v64 * v64))
    t = s * np.abs(v64) / norm
    p = t - np.floor(t)
    return norm, t, p


class Sums:
    """Per-coordinate and per-seed sums over a sweep of seeds."""

    def __init__(self, n):
        self.k1 = np.zeros(n, dtype=np.float64)   # sum of |k_i|
        self.q1 = np.zeros(n, dtype=np.float64)   # sum of Q_i
        self.err = []                              # ||Q - v||^2 per seed
        self.support = []                          # ||Q||_0 per seed
        self.count = 0

    def add_levels(self, v64, levels, norm_sent, s):
        k = levels.astype(np.float64)
        q = (float(norm_sent) / s) * k
        self.k1 += np.abs(k)
        self.q1 += q
        self.err.append(float(np.sum((q - v64) ** 2)))
        self.support.append(int(np.count_nonzero(levels)))
        self.count += 1

    def merge(self, other):
        self.k1 += other.k1
        self.q1 += other.q1
        self.err += other.err
        self.support += other.support
        self.count += other.count


def _sweep_quantize(args):
    v, s, seeds, source = args
    v64 = v.astype(np.float64)
    out = Sums(v.size)
    if source == "oracle":
        import oracle

        o = oracle.default()
        for seed in seeds:
            levels, norms, _ = o.quantize(v, v.size, s, seed)
            out.add_levels(v64, levels, norms[0], s)
    return out


def sweep(v: np.ndarray, s: int, seeds, processes: int = 8) -> Sums:
    """Quantises the single-bucket vector v with every seed (oracle, spawn pool)."""
    seeds = list(seeds)
    chunks = [seeds[i::processes] for i in range(processes)]
    ctx = mp.get_context("spawn")
    with ctx.Pool(processes) as pool:
        parts = pool.map(_sweep_quantize, [(v, s, c, "oracle") for c in chunks])
    total = Sums(v.size)
    for p in parts:
        total.merge(p)
    return total


def check_unbiased(v, s, sums: Sums, max_beyond_4se=20, max_abs_z=6.5):
    """|mean k_i - t_i| within 4 standard errors, counted over coordinates."""
    norm, t, p = exact_moments(v, s)
    N = sums.count
    var = p * (1.0 - p)
    mean_k = sums.k1 / N
    live = var * N >= 10.0  # normal approximation of the mean holds
    z = (mean_k[live] - t[live]) / np.sqrt(var[live] / N)
    dead = ~live
    # coordinates with p = 0 are exact; the other near-deterministic ones are
    # checked together: sum of (count - N t) within 4 SE of 0
    exact = p == 0.0
    assert np.all(mean_k[exact] == t[exact])
    few = dead & ~exact
    dev = float(np.sum((mean_k[few] - t[few]) * N))
    assert abs(dev) <= 4 * np.sqrt(float(np.sum(var[few] * N))) + 1.0, dev
    beyond = int(np.sum(np.abs(z) > 4.0))
    assert beyond <= max_beyond_4se, beyond
    assert float(np.max(np.abs(z))) < max_abs_z, float(np.max(np.abs(z)))
    # aggregate: mean z within 4 SE of 0 and mean z^2 within 4 SE of 1
    m = z.size
    assert abs(float(np.mean(z))) < 4.0 / np.sqrt(m)
    assert abs(float(np.mean(z * z)) - 1.0) < 4.0 * np.sqrt(2.0 / m) + 0.01
    # value domain: E[Q_i] = v_i
    qmean = sums.q1 / N
    zq = (qmean[live] - v[live]) / ((norm / s) * np.sqrt(var[live] / N))
    assert int(np.sum(np.abs(zq) > 4.0)) <= max_beyond_4se
    return beyond, float(np.max(np.abs(z)))


def check_variance(v, s, sums: Sums):
    norm, t, p = exact_moments(v, s)
    n = v.size
    closed = (norm ** 2 / s ** 2) * float(np.sum(p * (1 - p)))
    err = np.asarray(sums.err)
    measured = float(err.mean())
    se = float(err.std(ddof=1) / np.sqrt(err.size))
    assert abs(measured - closed) <= 4 * se, (measured, closed, se)
    bound = min(n / s ** 2, np.sqrt(n) / s) * norm ** 2
    assert measured <= bound
    return measured, closed, bound


def check_support(v, s, sums: Sums):
    norm, t, p = exact_moments(v, s)
    n = v.size
    expect = float(np.sum(np.where(t >= 1.0, 1.0, p)))
    sup = np.asarray(sums.support, dtype=np.float64)
    se = float(sup.std(ddof=1) / np.sqrt(sup.size))
    assert abs(sup.mean() - expect) <= 4 * se + 1e-9, (sup.mean(), expect, se)
    bound = s ** 2 + s * np.sqrt(n)
    assert sup.mean() <= bound
    return float(sup.mean()), expect, bound

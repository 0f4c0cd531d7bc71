"""Pins of the oracle's error-feedback wrapper (CPU).

"Sparsified SGD with Memory" (abstract): a compressor with error compensation keeps
the accumulated error of what it did not send in memory.  Around the QSGD codec this
reads: p = e + g, send Q(p), keep e <- p - Q(p) (Q(p) as a receiver decodes it; a
coordinate with no record keeps p).  The learning rate is left to the caller, which
scales g before the call.

Pins: hand-derived steps whose levels are exact; a case whose two possible outcomes
per coordinate are known in closed form, with their mean; the telescoping identity
sum_t Q(p_t) + e_T = e_0 + sum_t g_t within the fp32 rounding of the two adds of
each step; reduction to the plain encoder when e = 0; the same for the b-bit codes
and the max-norm scale."""

import numpy as np
import pytest

from quantized_gradient_compression_b200 import workloads as W

f32 = np.float32


def test_exact_levels_leave_no_error(oracle_lib):
    # g = (1, 4, 0..), e = (2, 0, ..): p = (3, 4, 0..), ||p|| = 5 = s, so t = (3, 4)
    # exactly and Q(p) = p: the memory ends at +0 everywhere
    g = np.array([1, 4, 0, 0, 0, 0, 0, 0], f32)
    e = np.array([2, 0, 0, 0, 0, 0, 0, 0], f32)
    for seed in (0, 7, 2**40 + 3):
        words, offsets, norms, st, e_new = oracle_lib.encode_ef(g, e, 8, 5, seed)
        pw, po, pn, _ = oracle_lib.encode(g + e, 8, 5, seed)
        assert st == 0 and norms.tolist() == [5.0]
        assert np.array_equal(words, pw) and np.array_equal(offsets, po)
        q, _ = oracle_lib.decode(words, offsets, 8, 8, 5)
        assert q.tolist() == [3, 4, 0, 0, 0, 0, 0, 0]
        assert e_new.view(np.uint32).tolist() == [0] * 8  # +0, not -0


def test_two_outcomes_per_coordinate(oracle_lib):
    # p = (-3, 4, 0, 0) with s = 1: ||p|| = 5, each non-zero coordinate rounds to
    # level 0 or 1 of step 5.  Coordinate 0: e_new = -3 (k = 0) or -3 - (-5) = 2;
    # coordinate 1: 4 or 4 - 5 = -1.  The mean of e_new is p - E[Q(p)] = 5 (p/5 - t).
    g = np.array([-3, 4, 0, 0], f32)
    e = np.zeros(4, f32)
    seen0, seen1, tot = set(), set(), np.zeros(4)
    N = 4000
    for seed in range(N):
        _, _, _, st, e_new = oracle_lib.encode_ef(g, e, 4, 1, seed)
        assert st == 0
        assert e_new[0] in (-3.0, 2.0) and e_new[1] in (4.0, -1.0) and not e_new[2:].any()
        seen0.add(float(e_new[0]))
        seen1.add(float(e_new[1]))
        tot += e_new
    assert seen0 == {-3.0, 2.0} and seen1 == {4.0, -1.0}
    t = np.array([f32(3) * f32(f32(1) / f32(5)), f32(4) * f32(f32(1) / f32(5))], np.float64)
    mean_expect = np.array([-3 + 5 * t[0], 4 - 5 * t[1]])
    se = 5 * np.sqrt(t * (1 - t) / N)
    assert np.all(np.abs(tot[:2] / N - mean_expect) <= 4 * se)


def _telescoping(steps, encode_step, decode_step):
    n = steps[0].size
    e = np.zeros(n, f32)
    e[::3] = W.normal(n, 99)[::3] * f32(0.01)
    e0 = e.astype(np.float64)
    sum_q = np.zeros(n)
    sum_g = np.zeros(n)
    bound = np.zeros(n)
    for t, g in enumerate(steps):
        p = (e + g).astype(f32)
        e = encode_step(g, e, t)
        q = decode_step(t)
        sum_q += q.astype(np.float64)
        sum_g += g.astype(np.float64)
        # each step rounds p = fl(e + g) and e = fl(p - q): half an ulp each
        bound += (np.abs(p.astype(np.float64)) + np.abs(e.astype(np.float64))) * 2.0**-24
    resid = np.abs(sum_q + e.astype(np.float64) - e0 - sum_g)
    assert np.all(resid <= bound * 1.0000001 + 1e-45), float(np.max(resid - bound))
    return e


@pytest.mark.parametrize("d,s", [(128, 4), (100, 1), (512, 16)])
def test_telescoping_elias(oracle_lib, d, s):
    steps = [W.normal(2000, 10 + t) for t in range(6)]
    streams = {}

    def enc(g, e, t):
        words, offsets, _, st, e_new = oracle_lib.encode_ef(g, e, d, s, seed=t)
        assert st == 0
        streams[t] = (words, offsets)
        return e_new

    def dec(t):
        return oracle_lib.decode(*streams[t], 2000, d, s)[0]

    e = _telescoping(steps, enc, dec)
    assert np.all(np.isfinite(e))


@pytest.mark.parametrize("b", [2, 4, 8])
def test_telescoping_bbit(oracle_lib, b):
    d = 128
    steps = [W.layered(1500, 20 + t) for t in range(5)]
    codes = {}

    def enc(g, e, t):
        c, nrm, st, e_new = oracle_lib.bbit_encode_ef(g, e, d, b, seed=t)
        assert st == 0
        codes[t] = (nrm, c)
        return e_new

    def dec(t):
        return oracle_lib.bbit_decode(*codes[t], 1500, d, b)[0]

    _telescoping(steps, enc, dec)


def test_error_is_below_one_level_step(oracle_lib):
    # |p_i - Q(p)_i| < fl(norm/s) (1 + 2^-22) wherever a record was sent: the error is
    # the rounding of t to a neighbouring level
    g = W.normal(4096, 5)
    e = W.normal(4096, 6) * f32(0.1)
    d, s = 256, 8
    words, offsets, norms, _, e_new = oracle_lib.encode_ef(g, e, d, s, seed=3)
    q, _ = oracle_lib.decode(words, offsets, g.size, d, s)
    step = np.repeat(norms.astype(np.float64) / s, d)[: g.size]
    sent = q != 0
    assert np.all(np.abs(e_new[sent].astype(np.float64)) < step[sent] * (1 + 2.0**-22))


def test_zero_memory_is_the_plain_encoder(oracle_lib):
    g = W.heavy_tailed_sparse(5000, 4)
    g[::17] = f32(-0.0)
    e = np.zeros_like(g)
    words, offsets, norms, st, e_new = oracle_lib.encode_ef(g, e, 512, 16, seed=11)
    pw, po, pn, pst = oracle_lib.encode(g, 512, 16, seed=11)
    assert st == pst and np.array_equal(words, pw) and np.array_equal(offsets, po)
    assert np.array_equal(norms.view(np.uint32), pn.view(np.uint32))
    q, _ = oracle_lib.decode(pw, po, g.size, 512, 16)
    unsent = q == 0
    # no record: the memory holds p = +0 + g, which is g except that -0 becomes +0
    assert np.array_equal(e_new[unsent], g[unsent])


def test_max_norm_scale_of_p(oracle_lib):
    g = W.normal(3000, 8)
    e = W.normal(3000, 9) * f32(0.5)
    p = (e + g).astype(f32)
    words, offsets, norms, st, _ = oracle_lib.encode_ef(g, e, 100, 4, seed=5, max_norm=True)
    mx = oracle_lib.maxnorms(p, 100)
    pw, po, _, _ = oracle_lib.encode(p, 100, 4, seed=5, norms_in=mx)
    assert np.array_equal(norms.view(np.uint32), mx.view(np.uint32))
    assert np.array_equal(words, pw) and np.array_equal(offsets, po)
    codes, bn, _, _ = oracle_lib.bbit_encode_ef(g, e, 100, 4, seed=5, max_norm=True)
    pc, pbn, _ = oracle_lib.bbit_encode(p, 100, 4, seed=5, norms_in=mx)
    assert np.array_equal(codes, pc) and np.array_equal(bn.view(np.uint32), mx.view(np.uint32))


def test_bbit_golden_step(oracle_lib):
    # b = 4 (s = 7): g = (0, -4, 0..), e = (0, -3, 0..): p = (0, -7, 0..), code 1111 at
    # bits 4..7 (word 0x0F000000) and no error left
    g = np.array([0, -4, 0, 0, 0, 0, 0, 0], f32)
    e = np.array([0, -3, 0, 0, 0, 0, 0, 0], f32)
    codes, norms, st, e_new = oracle_lib.bbit_encode_ef(g, e, 8, 4, seed=2)
    assert st == 0 and [int(c) for c in codes] == [0x0F000000] and norms.tolist() == [7.0]
    assert e_new.view(np.uint32).tolist() == [0] * 8


def test_nonfinite_bucket_keeps_p(oracle_lib):
    g = W.normal(16, 2)
    g[3] = np.inf
    e = W.normal(16, 3)
    words, offsets, norms, st, e_new = oracle_lib.encode_ef(g, e, 8, 4, seed=0)
    assert st & 1 and norms[0] == 0
    p = (e + g).astype(f32)
    assert np.array_equal(e_new[:8], p[:8])  # nothing of bucket 0 was sent
    q, _ = oracle_lib.decode(words, offsets, 16, 8, 4)
    sent = q[8:] != 0
    assert np.array_equal(e_new[8:][~sent], p[8:][~sent])

"""Pins of the oracle's mean of K received streams (CPU).

The definition paragraph places QSGD in distributed data-parallel optimisation: every
node quantises its gradient, the encodings are exchanged, and each node's update is
the mean of the K decoded gradients.  Reading: the sum of the decoded values left to
right from +0 (the decode-accumulate order), then one fp32 division by K."""

import numpy as np
import pytest

from helpers import bits_to_words
from quantized_gradient_compression_b200 import workloads as W

f32 = np.float32


def test_hand_values(oracle_lib):
    # stream a: norm 5, s = 5, levels (3, 4) -> (3, 4); stream b: norm 2, levels
    # (0, -1) -> (0, -0.4): the mean is (1.5, fl(4 - 0.4) / 2)
    a = bits_to_words("01000000101000000000000000000000" + "00110" + "00101000")
    b = bits_to_words("01000000000000000000000000000000" + "100" + "1" + "0")
    out, st = oracle_lib.decode_mean([(a, np.array([0, 45], np.uint64)), (b, np.array([0, 37], np.uint64))],
                                     2, 2, 5)
    assert st == 0
    assert out.tolist() == [1.5, float(f32(f32(4) + f32(-0.4)) / f32(2))]


def test_one_stream_is_the_decoder(oracle_lib):
    v = W.layered(5000, 3)
    w, o, _, _ = oracle_lib.encode(v, 512, 16, 4)
    ref, _ = oracle_lib.decode(w, o, v.size, 512, 16)
    out, st = oracle_lib.decode_mean([(w, o)], v.size, 512, 16)
    assert st == 0 and np.array_equal(out.view(np.uint32), ref.view(np.uint32))


def test_two_equal_streams_average_to_one(oracle_lib):
    # (q + q) / 2 = q exactly: doubling and halving are exact in binary
    v = W.normal(3000, 5)
    w, o, _, _ = oracle_lib.encode(v, 100, 7, 8)
    ref, _ = oracle_lib.decode(w, o, v.size, 100, 7)
    out, _ = oracle_lib.decode_mean([(w, o), (w, o)], v.size, 100, 7)
    assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("K", [3, 5, 8])
def test_mean_is_within_rounding_of_the_exact_mean(oracle_lib, K):
    # K - 1 adds and one division, each within half an ulp of its result
    n, d, s = 4000, 256, 8
    qs, streams = [], []
    for j in range(K):
        w, o, _, _ = oracle_lib.encode(W.normal(n, 40 + j), d, s, j)
        streams.append((w, o))
        qs.append(oracle_lib.decode(w, o, n, d, s)[0].astype(np.float64))
    out, _ = oracle_lib.decode_mean(streams, n, d, s)
    exact = np.sum(qs, axis=0) / K
    partial = np.abs(np.cumsum(qs, axis=0)).sum(axis=0)
    bound = (partial / K + np.abs(exact)) * 2.0**-24 * 1.0000001 + 1e-45
    assert np.all(np.abs(out.astype(np.float64) - exact) <= bound)


def test_mean_is_unbiased(oracle_lib):
    # E[mean_j Q(v_j)] = mean_j v_j: per coordinate within 4 standard errors over seeds
    n, d, s, K, N = 512, 512, 4, 4, 1500
    vs = [W.normal(n, 70 + j) for j in range(K)]
    target = np.mean([v.astype(np.float64) for v in vs], axis=0)
    acc = np.zeros(n)
    acc2 = np.zeros(n)
    for seed in range(N):
        streams = []
        for j, v in enumerate(vs):
            w, o, _, _ = oracle_lib.encode(v, d, s, seed * K + j)
            streams.append((w, o))
        out, _ = oracle_lib.decode_mean(streams, n, d, s)
        acc += out
        acc2 += out.astype(np.float64) ** 2
    mean = acc / N
    var = np.maximum(acc2 / N - mean**2, 1e-30)
    z = np.abs(mean - target) / np.sqrt(var / N)
    assert np.sum(z > 4) <= 3


def test_bbit_mean(oracle_lib):
    n, d, b = 2000, 128, 4
    streams, qs = [], []
    for j in range(3):
        c, nr, _ = oracle_lib.bbit_encode(W.normal(n, 10 + j), d, b, j)
        streams.append((nr, c))
        qs.append(oracle_lib.bbit_decode(nr, c, n, d, b)[0])
    out, st = oracle_lib.bbit_decode_mean(streams, n, d, b)
    ref = ((f32(0) + qs[0] + qs[1]).astype(f32) + qs[2]).astype(f32) / f32(3)
    assert st == 0 and np.array_equal(out.view(np.uint32), ref.astype(f32).view(np.uint32))
    one, _ = oracle_lib.bbit_decode_mean(streams[:1] * 2, n, d, b)
    assert np.array_equal(one.view(np.uint32), qs[0].view(np.uint32))

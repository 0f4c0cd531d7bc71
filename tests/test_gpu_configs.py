"""The benchmark workloads at full size, through the same C-ABI calls bench.py
times.  c1-c4: whole-vector parity with the oracle.  c5 (2^30 coordinates): every
bucket against the oracle, in slices of buckets checked by a pool of threads (the
oracle's C calls release the GIL), so that host memory stays bounded."""

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

from gpu_common import check_parity, device_vector, extract_bits, gpu_decode, gpu_encode, stream_norms, check_norms
from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [W.C1, W.C2, W.C3], ids=lambda w: w.name)
def test_full_config_parity(oracle_lib, w):
    check_parity(oracle_lib, w.generate(), w.d, w.s, w.seed)


def test_c4_receiver_aggregation(oracle_lib):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    senders = W.c4_streams()
    n, d, s = senders[0].n, senders[0].d, senders[0].s
    encs, host_streams = [], []
    for w in senders:
        v = w.generate()
        enc, words, offsets, status = gpu_encode(device_vector(v), d, s, w.seed)
        assert status == 0
        gnorms = stream_norms(words, offsets)
        _, _, onorms, _ = oracle_lib.encode(v, d, s, w.seed)
        check_norms(gnorms, onorms)
        r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, w.seed, norms_in=gnorms)
        assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)
        encs.append(enc)
        host_streams.append((words, offsets))
    base = W.normal(n, 999)
    acc = torch.from_numpy(base.copy()).cuda()
    _, st = B.decode_accumulate(encs, acc)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = base.copy()
    _, rst = oracle_lib.decode_accumulate(host_streams, n, d, s, ref)
    assert rst == 0
    assert np.array_equal(acc.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.fixture(scope="module")
def c5_input():
    return W.c5(1).generate()


@pytest.mark.parametrize("s", [1, 4, 16, 256])
def test_c5_full(oracle_lib, c5_input, s):
    """All 2,097,152 buckets: the stream bits, every offset and every decoded fp32
    against the oracle re-quantising with the GPU's norms (each norm first checked
    within 1e-6 of the oracle's own)."""
    import torch

    w = W.c5(s)
    v = c5_input
    n, d = v.size, w.d
    x = torch.from_numpy(v).cuda()
    enc, words, offsets, status = gpu_encode(x, d, s, w.seed)
    del x
    assert status == 0
    out, st = gpu_decode(enc)
    del enc
    torch.cuda.empty_cache()
    assert st == 0
    nb = (n + d - 1) // d
    assert offsets.size == nb + 1 and offsets[0] == 0
    per = 1 << 15  # buckets per slice

    def check(b0):
        b1 = min(nb, b0 + per)
        w0 = int(offsets[b0]) >> 5
        sub = words[w0:(int(offsets[b1]) >> 5) + 1]  # the slice's words
        gn = stream_norms(sub, offsets[b0:b1 + 1] - np.uint64(32 * w0))
        _, _, onorms, ost = oracle_lib.encode_range(v, d, s, w.seed, b0, b1)
        assert ost == 0
        check_norms(gn, onorms)
        rw, ro, _, rst = oracle_lib.encode_range(v, d, s, w.seed, b0, b1, norms_in=gn)
        assert rst == 0
        assert np.array_equal(ro, offsets[b0:b1 + 1] - offsets[b0])
        assert np.array_equal(rw, extract_bits(sub, int(offsets[b0]) - 32 * w0, int(offsets[b1]) - 32 * w0))
        c0, c1 = b0 * d, min(n, b1 * d)
        ref, dst = oracle_lib.decode(rw, ro, c1 - c0, d, s)
        assert dst == 0
        assert np.array_equal(out[c0:c1].view(np.uint32), ref.view(np.uint32))
        return b1 - b0

    with ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1))) as ex:
        assert sum(ex.map(check, range(0, nb, per))) == nb
    bits_per_coord = int(offsets[-1]) / n
    expect = {1: 0.45, 4: 1.10, 16: 2.38, 256: 8.28}[s]
    assert abs(bits_per_coord - expect) < 0.05 * expect + 0.02

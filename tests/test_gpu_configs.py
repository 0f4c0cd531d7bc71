"""The benchmark workloads at full size, through the same C-ABI calls bench.py
times.  c1-c4: whole-vector parity with the oracle.  c5 (2^30 coordinates): sampled
buckets against the oracle plus properties of the whole stream."""

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
def test_c5_sampled(oracle_lib, c5_input, s):
    import torch

    w = W.c5(s)
    v = c5_input
    n, d = v.size, w.d
    x = torch.from_numpy(v).cuda()
    enc, words, offsets, status = gpu_encode(x, d, s, w.seed)
    del x
    assert status == 0
    nb = (n + d - 1) // d
    assert offsets.size == nb + 1 and offsets[0] == 0
    sizes = np.diff(offsets.astype(np.int64))
    assert np.all(sizes >= 32) and np.all(sizes <= 32 + d * (2 + oracle_lib.omega_len(s)))
    out, st = gpu_decode(enc)
    assert st == 0
    rng = np.random.default_rng(s)
    picks = np.unique(np.concatenate([[0, 1, nb // 2, nb - 2, nb - 1], rng.integers(0, nb, 59)]))
    gn = stream_norms(words, offsets)
    for b in picks:
        b = int(b)
        vb = v[b * d:(b + 1) * d]
        onorm = oracle_lib.bucket_norm(vb)
        check_norms(gn[b:b + 1], np.array([onorm], np.float32))
        ref_words, ref_bits, _ = oracle_lib.encode_bucket(vb, b * d, s, w.seed, norm_in=gn[b])
        begin, end = int(offsets[b]), int(offsets[b + 1])
        assert ref_bits == end - begin
        assert np.array_equal(extract_bits(words, begin, end), ref_words[:(ref_bits + 31) // 32])
        ref_out, rst = oracle_lib.decode_bucket(words, begin, end, vb.size, s)
        assert rst == 0
        assert np.array_equal(out[b * d:(b + 1) * d].view(np.uint32), ref_out.view(np.uint32))
    bits_per_coord = int(offsets[-1]) / n
    expect = {1: 0.45, 4: 1.10, 16: 2.38, 256: 8.28}[s]
    assert abs(bits_per_coord - expect) < 0.05 * expect + 0.02

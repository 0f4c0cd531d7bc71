"""The mean of K streams and the data-parallel exchange through the C ABI (GPU).

qsgd_decode_mean and qsgd_bbit_decode_mean run on oracle-made streams and are compared
with the oracle's mean bit for bit, at K = 1 up to K > 16 (more than one accumulate
launch), for general shapes and a misaligned output.  The exchange runs once through an
NCCL process group of one rank: every collective of the step runs on the device.  The
K-stream layout of the library codec is checked on K streams gathered by hand."""

import numpy as np
import pytest

from gpu_common import device_vector
from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _streams(o, K, n, d, s, seed0=0):
    out = []
    for j in range(K):
        w, off, _, _ = o.encode(W.layered(n, 200 + j) * np.float32(2.0 ** (j % 5)), d, s, seed0 + j)
        out.append((w, off))
    return out


@pytest.mark.parametrize("K,n,d,s,mis", [(1, 100_000, 512, 16, 0), (2, 100_000, 512, 16, 0),
                                         (3, 60_001, 100, 7, 0), (8, 200_003, 512, 4, 0),
                                         (17, 30_000, 256, 16, 0), (5, 40_000, 512, 16, 1)])
def test_decode_mean_bit_exact(oracle_lib, K, n, d, s, mis):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    streams = _streams(oracle_lib, K, n, d, s)
    dev = [(torch.from_numpy(np.concatenate([w, np.zeros(1, np.uint32)]).view(np.int32)).cuda(),
            torch.from_numpy(off.view(np.int64)).cuda()) for w, off in streams]
    out = device_vector(np.full(n, np.nan, np.float32), mis)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = B.qsgd_decode_mean([w.data_ptr() for w, _ in dev], [w.numel() for w, _ in dev],
                            [o.data_ptr() for _, o in dev], K, n, d, s, out.data_ptr(), st.data_ptr(),
                            torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    ref, rst = oracle_lib.decode_mean(streams, n, d, s)
    assert int(st.item()) == 0 and rst == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("K,n,d,b", [(1, 50_000, 512, 4), (3, 100_003, 512, 2), (8, 60_000, 100, 8)])
def test_bbit_decode_mean_bit_exact(oracle_lib, K, n, d, b):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    streams, dev = [], []
    for j in range(K):
        c, nr, _ = oracle_lib.bbit_encode(W.normal(n, 300 + j), d, b, j)
        streams.append((nr, c))
        dev.append((torch.from_numpy(nr.copy()).cuda(),
                    torch.from_numpy(np.concatenate([c, np.zeros(1, np.uint32)]).view(np.int32)).cuda()))
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert B.qsgd_bbit_decode_mean([x.data_ptr() for x, _ in dev], [c.data_ptr() for _, c in dev], K, n, d, b,
                                   out.data_ptr(), st.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    ref, _ = oracle_lib.bbit_decode_mean(streams, n, d, b)
    assert int(st.item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_library_codec_layout(oracle_lib):
    """K streams gathered rank-major and padded to the longest, as the exchange lays them
    out, decode to the oracle's mean."""
    import torch
    from quantized_gradient_compression_b200 import exchange as X

    n, d, s, K = 80_000, 512, 16, 4
    codec = X.LibraryCodec(n, d, s, "cuda")
    streams = _streams(oracle_lib, K, n, d, s, seed0=11)
    maxw = max((int(off[-1]) + 31) // 32 for _, off in streams)
    g_words = torch.zeros(K * maxw, dtype=torch.int32, device="cuda")
    g_off = torch.zeros(K * (codec.nb + 1), dtype=torch.int64, device="cuda")
    for j, (w, off) in enumerate(streams):
        g_words[j * maxw:j * maxw + w.size] = torch.from_numpy(w.view(np.int32)).cuda()
        g_off[j * (codec.nb + 1):(j + 1) * (codec.nb + 1)] = torch.from_numpy(off.view(np.int64)).cuda()
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    codec.decode_mean(g_words, maxw, g_off, K, out)
    torch.cuda.synchronize()
    ref, _ = oracle_lib.decode_mean(streams, n, d, s)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_exchange_on_one_nccl_rank(oracle_lib):
    """One NCCL rank: the step's three gathers run on the device, and the mean of one
    stream is its decode.  With the memory, the stream and memory match the oracle's
    error-feedback encode."""
    import datetime

    import torch
    import torch.distributed as dist
    from gpu_common import stream_norms
    from quantized_gradient_compression_b200 import exchange as X

    n, d, s = 100_003, 512, 16
    store = dist.HashStore()
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x = X.EliasExchange(X.LibraryCodec(n, d, s, "cuda"))
        g = W.layered(n, 5)
        out = x.step(device_vector(g), seed=9)
        torch.cuda.synchronize()
        words = x.codec.words[: x.last.max_words].cpu().numpy().view(np.uint32)
        offsets = x.codec.offsets.cpu().numpy().view(np.uint64)
        gn = stream_norms(words, offsets)
        r_words, r_off, _, _ = oracle_lib.encode(g, d, s, X.rank_seed(9, 0), norms_in=gn)
        assert np.array_equal(words[: r_words.size], r_words) and np.array_equal(offsets, r_off)
        ref, _ = oracle_lib.decode(r_words, r_off, n, d, s)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        # with the error-feedback memory, two steps
        mem = torch.zeros(n, dtype=torch.float32, device="cuda")
        e_ref = np.zeros(n, np.float32)
        for t in range(2):
            g = W.layered(n, 20 + t)
            out = x.step(device_vector(g), seed=30 + t, memory=mem)
            torch.cuda.synchronize()
            words = x.codec.words[: x.last.max_words].cpu().numpy().view(np.uint32)
            offsets = x.codec.offsets.cpu().numpy().view(np.uint64)
            r_words, r_off, _, _, e_ref = oracle_lib.encode_ef(g, e_ref, d, s, X.rank_seed(30 + t, 0),
                                                               norms_in=stream_norms(words, offsets))
            assert np.array_equal(words[: r_words.size], r_words)
            assert np.array_equal(mem.cpu().numpy().view(np.uint32), e_ref.view(np.uint32))
            ref, _ = oracle_lib.decode(r_words, r_off, n, d, s)
            assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        # b-bit
        xb = X.BbitExchange(X.LibraryBbitCodec(n, d, 4, "cuda"))
        out = xb.step(device_vector(g), seed=4)
        torch.cuda.synchronize()
        norms = xb.codec.norms.cpu().numpy()
        c, _, _ = oracle_lib.bbit_encode(g, d, 4, X.rank_seed(4, 0), norms_in=norms)
        assert np.array_equal(xb.codec.codes.cpu().numpy().view(np.uint32)[: c.size], c)
        ref, _ = oracle_lib.bbit_decode(norms, c, n, d, 4)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    finally:
        dist.destroy_process_group()

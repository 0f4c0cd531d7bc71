"""Decode-accumulate through the C ABI against the oracle (GPU).

The streams are made by the oracle on the host and copied to the device, so the
decoders are checked on inputs that owe nothing to the CUDA encoder.  The receiver
buffer starts with ordinary values, exact zeros of both signs and values the
updates cancel; the sum is fp32 adds in stream order, so the comparison is
bit-exact."""

import numpy as np
import pytest

from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _base(n, seed):
    rng = np.random.default_rng(seed)
    b = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    b[rng.random(n) < 0.2] = np.float32(-0.0)
    b[rng.random(n) < 0.1] = np.float32(0.0)
    return b


# (n, d, s, K): the one-stream row decoder (K = 1), the several-stream decoders on
# d <= 1024 (byte codes side by side for s <= 127, fp32 tiles side by side below
# s = 1024, fp32 tiles one stream after another above), the large-bucket decoder
# (d > 1024), the one-lane decoders (d < 4 or d not a multiple of 4), and K beyond one
# launch's 16 streams
CASES = [
    (40_000, 132, 3, 3),
    (100_003, 512, 16, 1),
    (100_003, 512, 16, 3),
    (60_000, 512, 4, 17),
    (40_000, 512, 300, 3),
    (20_000, 512, 2000, 2),
    (50_000, 2048, 64, 2),
    (30_000, 100, 7, 3),
    (30_001, 8192, 2, 2),
    (20_000, 3, 5, 2),
]


@pytest.mark.parametrize("n,d,s,K", CASES, ids=["n%d-d%d-s%d-K%d" % c for c in CASES])
def test_accumulate_matches_oracle(oracle_lib, n, d, s, K):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    streams, dev = [], []
    for j in range(K):
        v = W.normal(n, 300 + j)
        words, offsets, _, st = oracle_lib.encode(v, d, s, seed=77 + j)
        assert st == 0
        streams.append((words, offsets))
        w = torch.from_numpy(np.concatenate([words, np.zeros(1, np.uint32)]).view(np.int32)).cuda()
        o = torch.from_numpy(offsets.view(np.int64).copy()).cuda()
        dev.append((w, o))
    base = _base(n, d + K)
    ref = base.copy()
    _, rst = oracle_lib.decode_accumulate(streams, n, d, s, ref)
    assert rst == 0

    out = torch.from_numpy(base.copy()).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = B.qsgd_decode_accumulate([w.data_ptr() for w, _ in dev], [w.numel() for w, _ in dev],
                                  [o.data_ptr() for _, o in dev], K, n, d, s, out.data_ptr(),
                                  status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("d", [512, 2048, 132])
def test_decode_of_oracle_streams(oracle_lib, d):
    """Plain decode of oracle-made streams (layered data: many buckets are nearly
    empty and some records need the bit-serial path)."""
    import torch
    from quantized_gradient_compression_b200 import binding as B

    n, s = 200_001, 16
    v = W.layered(n, 4)
    words, offsets, _, st = oracle_lib.encode(v, d, s, seed=9)
    ref, rst = oracle_lib.decode(words, offsets, n, d, s)
    assert st == 0 and rst == 0
    w = torch.from_numpy(np.concatenate([words, np.zeros(1, np.uint32)]).view(np.int32)).cuda()
    o = torch.from_numpy(offsets.view(np.int64).copy()).cuda()
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = B.qsgd_decode(w.data_ptr(), w.numel(), o.data_ptr(), n, d, s, out.data_ptr(), status.data_ptr(),
                       torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))

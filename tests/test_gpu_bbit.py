"""Fixed-width b-bit QSGD through the C ABI against the oracle (GPU).

Encoder: norms within 1e-6 of the oracle's; the oracle re-quantises with the GPU's
norms and its codes must equal the GPU's bit for bit.  Decoder and decode-accumulate:
bit-exact on oracle-made codes."""

import numpy as np
import pytest

from gpu_common import NORM_RTOL, device_vector
from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu

PAD = 1024
SENTINEL = np.uint32(0x7FC0DEAD)


def _gpu_encode(x, d, b, seed):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    enc = B.bbit_encode(x, d, b, seed)
    torch.cuda.synchronize()
    n = x.numel()
    norms = enc.norms.cpu().numpy()[: (n + d - 1) // d].copy()
    codes = enc.codes.cpu().numpy().view(np.uint32)[: B.qsgd_bbit_code_words(n, b)].copy()
    return enc, norms, codes, int(enc.status.item())


def _check_encode(oracle_lib, v, d, b, seed, misalign=0):
    x = device_vector(v, misalign)
    enc, gnorms, codes, st = _gpu_encode(x, d, b, seed)
    r_codes, r_norms, rst = oracle_lib.bbit_encode(v, d, b, seed)
    assert st == rst
    nz = r_norms != 0
    assert np.array_equal(gnorms == 0, ~nz)
    assert np.all(np.abs(gnorms[nz].astype(np.float64) - r_norms[nz]) <= NORM_RTOL * np.abs(r_norms[nz]))
    o_codes, o_norms, _ = oracle_lib.bbit_encode(v, d, b, seed, norms_in=gnorms)
    assert np.array_equal(o_norms.view(np.uint32), gnorms.view(np.uint32))
    assert np.array_equal(codes, o_codes)
    return enc, o_norms, o_codes


CASES = [
    # fast path: one warp per bucket, d = 128V
    ("layered", 1_000_003, 512, 2), ("layered", 1_000_003, 512, 4), ("layered", 1_000_003, 512, 8),
    ("normal", 200_000, 128, 2), ("normal", 200_000, 128, 4), ("normal", 200_000, 256, 2),
    ("normal", 300_001, 1024, 8), ("normal", 300_001, 1024, 2),
    # general path: bucket norms, then one thread per code word
    ("normal", 100_001, 100, 4), ("normal", 9_999, 3, 2), ("normal", 50_000, 384, 8),
    ("heavy_tailed_sparse", 200_000, 8192, 4), ("normal", 7, 512, 4), ("normal", 1, 1, 8),
]


@pytest.mark.parametrize("kind,n,d,b", CASES, ids=["%s-n%d-d%d-b%d" % c for c in CASES])
def test_bbit_parity(oracle_lib, kind, n, d, b):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    v = W.GENERATORS[kind](n, n % 89 + d + b)
    enc, norms, codes = _check_encode(oracle_lib, v, d, b, seed=99)
    out, st = B.bbit_decode(enc)
    torch.cuda.synchronize()
    ref, rst = oracle_lib.bbit_decode(norms, codes, n, d, b)
    assert int(st.item()) == 0 and rst == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("d,b", [(512, 4), (100, 2)])
def test_bbit_misaligned_input(oracle_lib, d, b):
    _check_encode(oracle_lib, W.normal(40_003, 3), d, b, seed=5, misalign=1)


def test_bbit_special_values(oracle_lib):
    v = W.normal(4096, 8)
    v[0:512] = 0.0                 # a zero bucket
    v[600] = np.inf                # a non-finite bucket
    v[1100] = np.nan
    v[1536:2048] = 1e-30           # tiny values: the rescaled norm
    v[2048:2560] = 3e38            # squares overflow: the rescaled norm
    for b in (2, 4, 8):
        for d in (512, 100):
            _check_encode(oracle_lib, v, d, b, seed=1)


@pytest.mark.parametrize("n,d,b,K", [(100_003, 512, 4, 3), (50_000, 100, 2, 2), (30_001, 1024, 8, 17)])
def test_bbit_decode_accumulate(oracle_lib, n, d, b, K):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    streams, dev = [], []
    for j in range(K):
        codes, norms, _ = oracle_lib.bbit_encode(W.normal(n, 500 + j), d, b, seed=j)
        streams.append((norms, codes))
        dev.append((torch.from_numpy(norms.copy()).cuda(),
                    torch.from_numpy(np.concatenate([codes, np.zeros(1, np.uint32)]).view(np.int32)).cuda()))
    base = W.normal(n, 7) * np.float32(1e-2)
    base[::5] = np.float32(-0.0)
    ref = base.copy()
    _, rst = oracle_lib.bbit_decode_accumulate(streams, n, d, b, ref)
    out = torch.from_numpy(base.copy()).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = B.qsgd_bbit_decode_accumulate([x.data_ptr() for x, _ in dev], [c.data_ptr() for _, c in dev], K, n, d, b,
                                       out.data_ptr(), st.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and rst == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def _decode_guarded(norms, codes, n, d, b):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    nt = torch.from_numpy(norms.copy()).cuda()
    ct = torch.from_numpy(np.concatenate([codes, np.zeros(1, np.uint32)]).view(np.int32)).cuda()
    buf = torch.from_numpy(np.full(n + 2 * PAD, SENTINEL, dtype=np.uint32).view(np.int32)).cuda()
    out = buf[PAD:PAD + n].view(torch.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert B.qsgd_bbit_decode(nt.data_ptr(), ct.data_ptr(), n, d, b, out.data_ptr(), st.data_ptr(),
                              torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    host = buf.cpu().numpy().view(np.uint32)
    assert np.all(host[:PAD] == SENTINEL) and np.all(host[PAD + n:] == SENTINEL)
    return host[PAD:PAD + n].view(np.float32), int(st.item())


@pytest.mark.parametrize("kind", ["sign_on_zero", "negative_norm", "nan_norm", "zero_norm_with_code",
                                  "underflowing_scale"])
@pytest.mark.parametrize("d", [512, 100])
def test_bbit_malformed_flagged(oracle_lib, kind, d):
    n, b = 4_001, 4
    codes, norms, _ = oracle_lib.bbit_encode(W.normal(n, 11), d, b, seed=2)
    bk = 3
    if kind == "sign_on_zero":
        # find a zero code in bucket bk and set its sign bit
        for i in range(bk * d, (bk + 1) * d):
            w, sh = divmod(i * b, 32)
            if (int(codes[w]) >> (32 - b - sh)) & ((1 << b) - 1) == 0:
                codes[w] |= np.uint32(1 << (31 - sh))
                break
    elif kind == "negative_norm":
        norms[bk] = -norms[bk]
    elif kind == "nan_norm":
        norms[bk] = np.nan
    elif kind == "zero_norm_with_code":
        norms[bk] = 0.0
    else:
        norms[bk] = np.uint32(1).view(np.float32)
    _, rst = oracle_lib.bbit_decode(norms, codes, n, d, b)
    out, st = _decode_guarded(norms, codes, n, d, b)
    assert rst & 2 and st & 2
    ref, _ = oracle_lib.bbit_decode(norms, codes, n, d, b)
    keep = np.ones(n, bool)
    keep[bk * d:(bk + 1) * d] = False
    assert np.array_equal(out[keep].view(np.uint32), ref[keep].view(np.uint32))

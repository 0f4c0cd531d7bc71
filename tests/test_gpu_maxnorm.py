"""The max-norm (QSGDinf) scale through the C ABI against the oracle (GPU).

A max is exact, so the GPU's sent norms must equal the oracle's bit for bit, and the
streams and codes must equal the oracle's with those norms."""

import numpy as np
import pytest

from gpu_common import device_vector
from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _special(n, seed):
    v = W.normal(n, seed)
    v[:512] = 0.0
    v[700] = np.inf
    v[1300] = np.nan
    v[1600:2048] = 1e-30
    v[2048:2200] = 3e38
    return v


CASES = [("layered", 600_001, 512, 16), ("normal", 100_000, 128, 8), ("normal", 100_000, 1024, 64),
         ("normal", 50_001, 100, 7), ("heavy_tailed_sparse", 200_000, 8192, 1), ("special", 10_000, 512, 16),
         ("special", 10_000, 100, 4)]


def _vec(kind, n):
    return _special(n, 3) if kind == "special" else W.GENERATORS[kind](n, n % 97)


@pytest.mark.parametrize("kind,n,d,s", CASES, ids=["%s-n%d-d%d-s%d" % c for c in CASES])
def test_elias_maxnorm_bit_exact(oracle_lib, kind, n, d, s):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    v = _vec(kind, n)
    enc = B.encode(device_vector(v), d, s, seed=31, norm_kind=B.QSGD_NORM_MAX)
    torch.cuda.synchronize()
    offsets = enc.offsets.cpu().numpy().view(np.uint64)
    words = enc.words[: (int(offsets[-1]) + 31) // 32].cpu().numpy().view(np.uint32)
    r_words, r_offsets, r_norms, rst = oracle_lib.encode(v, d, s, 31, norms_in=oracle_lib.maxnorms(v, d))
    assert int(enc.status.item()) == rst
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)
    out, st = B.decode(enc)
    torch.cuda.synchronize()
    ref, _ = oracle_lib.decode(r_words, r_offsets, n, d, s)
    assert int(st.item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("kind,n,d,b", [("layered", 300_001, 512, 4), ("normal", 100_000, 128, 2),
                                        ("normal", 50_001, 100, 8), ("special", 10_000, 512, 4),
                                        ("special", 10_000, 100, 2)])
def test_bbit_maxnorm_bit_exact(oracle_lib, kind, n, d, b):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    v = _vec(kind, n)
    enc = B.bbit_encode(device_vector(v), d, b, seed=17, norm_kind=B.QSGD_NORM_MAX)
    torch.cuda.synchronize()
    norms = enc.norms.cpu().numpy()[: (n + d - 1) // d]
    codes = enc.codes.cpu().numpy().view(np.uint32)[: B.qsgd_bbit_code_words(n, b)]
    r_codes, r_norms, rst = oracle_lib.bbit_encode(v, d, b, 17, norms_in=oracle_lib.maxnorms(v, d))
    assert int(enc.status.item()) == rst
    assert np.array_equal(norms.view(np.uint32), r_norms.view(np.uint32))
    assert np.array_equal(codes, r_codes)

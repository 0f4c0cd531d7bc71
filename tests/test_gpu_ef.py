"""Error feedback through the C ABI against the oracle (GPU).

p = e + g is encoded and the memory becomes p minus its decoded value ("Sparsified
SGD with Memory", abstract).  Under the L2 scale the oracle re-quantises with the
GPU's sent norms (the wire format lets an encoder choose its fp32 norm within 1e-6);
the stream, the codes and the new memory must then equal the oracle's bit for bit.
Under the max-norm scale nothing is taken from the GPU.  A NaN in p is compared as
a NaN: the GPU's adds give the canonical NaN, the host's keep the payload."""

import numpy as np
import pytest

from gpu_common import check_norms, device_vector, stream_norms
from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _same(a, b):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    nan = np.isnan(a) & np.isnan(b)
    return bool(np.array_equal(a.view(np.uint32)[~nan], b.view(np.uint32)[~nan]))


def _inputs(kind, n, seed):
    if kind == "special":
        g = W.normal(n, seed)
        g[:600] = 0.0
        g[700] = np.inf
        g[1300] = np.nan
        g[1600:2100] = 1e-30
        g[2100:2300] = 3e38
        g[2400:2600] = -0.0
        e = W.normal(n, seed + 1) * np.float32(0.01)
        e[:600] = 0.0
        e[2400:2600] = -0.0
        e[1700:1800] = 1e-38
        return g, e
    g = W.GENERATORS[kind](n, seed)
    e = W.GENERATORS[kind](n, seed + 7) * np.float32(0.05)
    return g, e


def _gpu_ef(g, e, d, s, seed, norm_kind, misalign_g=0, misalign_e=0):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    xg = device_vector(g, misalign_g)
    xe = device_vector(e, misalign_e)
    enc = B.encode_ef(xg, xe, d, s, seed, norm_kind=norm_kind)
    torch.cuda.synchronize()
    offsets = enc.offsets.cpu().numpy().view(np.uint64).copy()
    words = enc.words[: (int(offsets[-1]) + 31) // 32].cpu().numpy().view(np.uint32).copy()
    assert np.array_equal(xg.cpu().numpy().view(np.uint32), g.view(np.uint32))  # g is read only
    return words, offsets, int(enc.status.item()), xe.cpu().numpy()


def _check_elias(o, g, e, d, s, seed, norm_kind, **mis):
    from quantized_gradient_compression_b200 import binding as B

    words, offsets, st, e_new = _gpu_ef(g, e, d, s, seed, norm_kind, **mis)
    if norm_kind == B.QSGD_NORM_MAX:
        r = o.encode_ef(g, e, d, s, seed, max_norm=True)
        r_st = r[3]
    else:
        # the status comes from the oracle's own norms: a bucket re-quantised with a
        # sent norm of 0 cannot tell why it was sent as zero
        own = o.encode_ef(g, e, d, s, seed)
        gn = stream_norms(words, offsets)
        check_norms(gn, own[2])
        r_st = own[3]
        r = o.encode_ef(g, e, d, s, seed, norms_in=gn)
    r_words, r_offsets, _, _, r_e = r
    assert st == r_st
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)
    assert _same(e_new, r_e)
    return e_new


CASES = [
    # one fused pass: the fast encoder shapes, both arrays 16-byte aligned
    ("layered", 600_001, 512, 16, 0, 0), ("normal", 100_000, 128, 4, 0, 0), ("normal", 100_003, 1024, 1, 0, 0),
    ("normal", 50_000, 256, 64, 0, 0), ("special", 10_000, 512, 16, 0, 0),
    # three passes: general shapes, or a misaligned array
    ("normal", 50_001, 100, 7, 0, 0), ("heavy_tailed_sparse", 200_000, 8192, 1, 0, 0),
    ("layered", 100_000, 512, 16, 1, 0), ("layered", 100_000, 512, 16, 0, 3), ("special", 10_000, 100, 4, 0, 0),
    ("normal", 7, 512, 4, 0, 0), ("normal", 1, 1, 1, 0, 0),
]


@pytest.mark.parametrize("norm", ["l2", "max"])
@pytest.mark.parametrize("kind,n,d,s,mg,me", CASES, ids=["%s-n%d-d%d-s%d-g%d-e%d" % c for c in CASES])
def test_elias_ef_bit_exact(oracle_lib, kind, n, d, s, mg, me, norm):
    from quantized_gradient_compression_b200 import binding as B

    g, e = _inputs(kind, n, n % 53)
    nk = B.QSGD_NORM_MAX if norm == "max" else B.QSGD_NORM_L2
    _check_elias(oracle_lib, g, e, d, s, 41, nk, misalign_g=mg, misalign_e=me)


@pytest.mark.parametrize("d,s,mg", [(512, 16, 0), (100, 3, 0), (512, 4, 1)])
def test_elias_ef_steps_carry_memory(oracle_lib, d, s, mg):
    """Four steps, the memory carried on the GPU and in the oracle; each step must
    agree bit for bit, so the memories never drift apart."""
    n = 70_001
    e = np.zeros(n, np.float32)
    for t in range(4):
        g = W.layered(n, 300 + t)
        e = _check_elias(oracle_lib, g, e, d, s, t, 0, misalign_g=mg)


def test_elias_ef_empty():
    import torch
    from quantized_gradient_compression_b200 import binding as B

    g = torch.empty(0, dtype=torch.float32, device="cuda")
    e = torch.empty(0, dtype=torch.float32, device="cuda")
    enc = B.encode_ef(g, e, 512, 16, 0)
    torch.cuda.synchronize()
    assert int(enc.offsets[0].item()) == 0 and int(enc.status.item()) == 0


def _check_bbit(o, g, e, d, b, seed, norm_kind, misalign_g=0, misalign_e=0):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    n = g.size
    xg = device_vector(g, misalign_g)
    xe = device_vector(e, misalign_e)
    enc = B.bbit_encode_ef(xg, xe, d, b, seed, norm_kind=norm_kind)
    torch.cuda.synchronize()
    norms = enc.norms.cpu().numpy()[: (n + d - 1) // d].copy()
    codes = enc.codes.cpu().numpy().view(np.uint32)[: B.qsgd_bbit_code_words(n, b)].copy()
    e_new = xe.cpu().numpy()
    if norm_kind == B.QSGD_NORM_MAX:
        r_codes, r_norms, r_st, r_e = o.bbit_encode_ef(g, e, d, b, seed, max_norm=True)
        assert np.array_equal(norms.view(np.uint32), r_norms.view(np.uint32))
    else:
        _, own_norms, r_st, _ = o.bbit_encode_ef(g, e, d, b, seed)  # status from the oracle's own norms
        check_norms(norms, own_norms)
        r_codes, r_norms, _, r_e = o.bbit_encode_ef(g, e, d, b, seed, norms_in=norms)
    assert int(enc.status.item()) == r_st
    assert np.array_equal(codes, r_codes)
    assert _same(e_new, r_e)
    return e_new


BCASES = [("layered", 300_001, 512, 4, 0, 0), ("normal", 100_000, 128, 2, 0, 0), ("normal", 100_003, 1024, 8, 0, 0),
          ("special", 10_000, 512, 4, 0, 0),
          ("normal", 50_001, 100, 8, 0, 0), ("normal", 60_000, 384, 2, 0, 0), ("layered", 80_000, 512, 4, 1, 0),
          ("layered", 80_000, 256, 2, 0, 2), ("special", 10_000, 100, 2, 0, 0)]


@pytest.mark.parametrize("norm", ["l2", "max"])
@pytest.mark.parametrize("kind,n,d,b,mg,me", BCASES, ids=["%s-n%d-d%d-b%d-g%d-e%d" % c for c in BCASES])
def test_bbit_ef_bit_exact(oracle_lib, kind, n, d, b, mg, me, norm):
    from quantized_gradient_compression_b200 import binding as B

    g, e = _inputs(kind, n, n % 59)
    nk = B.QSGD_NORM_MAX if norm == "max" else B.QSGD_NORM_L2
    _check_bbit(oracle_lib, g, e, d, b, 23, nk, misalign_g=mg, misalign_e=me)


def test_bbit_ef_steps_carry_memory(oracle_lib):
    n = 50_000
    e = np.zeros(n, np.float32)
    for t in range(4):
        e = _check_bbit(oracle_lib, W.normal(n, 900 + t), e, 512, 2, t, 0)


def test_ef_full_size_bench_workload(oracle_lib):
    """The benchmark's gradient (n = 25,557,032, d = 512, s = 16) through the fused
    call: stream and memory bit-exact against the oracle."""
    w = W.C2
    g = w.generate()
    e = W.small_normal(w.n, 77)
    _check_elias(oracle_lib, g, e, w.d, w.s, w.seed, 0)

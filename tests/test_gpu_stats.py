"""The page's distributional claims checked on the CUDA path (encode + decode on the
GPU, 10^4 seeds of the single-bucket n = 65,536 vector at s = sqrt(n) = 256)."""

import numpy as np
import pytest

import stats_common as sc
from quantized_gradient_compression_b200 import workloads

pytestmark = pytest.mark.gpu

SEEDS = 10_000


@pytest.fixture(scope="module")
def gpu_sweep():
    import torch
    from quantized_gradient_compression_b200 import binding as B

    v = workloads.C1.generate()
    n, s = v.size, 256
    x = torch.from_numpy(v).cuda()
    v64 = torch.from_numpy(v.astype(np.float64)).cuda()
    k1 = torch.zeros(n, dtype=torch.float64, device="cuda")
    q1 = torch.zeros(n, dtype=torch.float64, device="cuda")
    err, support, bits = [], [], []
    status = 0
    for seed in range(SEEDS):
        enc = B.encode(x, n, s, seed)
        out, st = B.decode(enc)
        q = out.double()
        norm = enc.words[0:1].view(torch.float32).double()  # the bucket's norm field (word 0)
        scale = (norm.float() / float(s)).double()
        k1 += torch.round(q.abs() / scale)
        q1 += q
        err.append(torch.sum((q - v64) ** 2))
        support.append(torch.count_nonzero(out))
        bits.append(enc.offsets[-1])
        if seed % 1000 == 999:
            status |= int(enc.status.item()) | int(st.item())
    torch.cuda.synchronize()
    sums = sc.Sums(n)
    sums.k1 = k1.cpu().numpy()
    sums.q1 = q1.cpu().numpy()
    sums.err = [float(e) for e in torch.stack(err).cpu()]
    sums.support = [int(c) for c in torch.stack(support).cpu()]
    sums.count = SEEDS
    return v, sums, np.array([int(b) for b in torch.stack(bits).cpu()]), status


def test_gpu_unbiased(gpu_sweep):
    v, sums, _, status = gpu_sweep
    assert status == 0
    sc.check_unbiased(v, 256, sums)


def test_gpu_variance(gpu_sweep):
    v, sums, _, _ = gpu_sweep
    sc.check_variance(v, 256, sums)


def test_gpu_support(gpu_sweep):
    v, sums, _, _ = gpu_sweep
    sc.check_support(v, 256, sums)


def test_gpu_bits_within_2_818n_plus_32(gpu_sweep):
    v, _, bits, _ = gpu_sweep
    n = v.size
    assert bits.mean() + 4 * bits.std(ddof=1) / np.sqrt(bits.size) <= 2.818 * n + 32

"""CUDA path vs oracle, element by element, through the C ABI (GPU)."""

import numpy as np
import pytest

from gpu_common import check_parity
from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu


def vec(kind, n, seed):
    return W.GENERATORS[kind](n, seed)


# (kind, n, d, s): several tiles and a ragged tail on every encoder and decoder path:
# the staged short coder (s <= 31, d <= 16384, one or several 512-coordinate chunks),
# the staged lane-strided coder (s > 31, d <= 1024), the one-pass coder (other shapes),
# the row decoder with byte codes (s <= 127) and 16-bit codes, the large-bucket
# decoder (d > 1024) and the one-lane decoders (d not a multiple of 4)
CASES = [
    ("layered", 2_000_001, 512, 16),       # fast path, ragged last bucket (129)
    ("layered", 1_000_000, 512, 16),
    ("normal", 300_000, 512, 1),
    ("normal", 300_000, 512, 4),
    ("normal", 300_000, 512, 256),
    ("small_normal", 500_000, 512, 4),
    ("normal", 100_000, 128, 8),           # fast path V = 1
    ("normal", 100_000, 256, 8),           # V = 2
    ("normal", 100_000, 1000, 8),          # V = 8, d not a power of two
    ("normal", 100_000, 1024, 16),         # V = 8, gap 1024 beyond the table
    ("normal", 100_001, 1025, 16),         # general path
    ("heavy_tailed_sparse", 1_000_000, 8192, 1),
    ("normal", 65_536, 65_536, 256),       # one bucket
    ("normal", 70_001, 4096, 2),
    ("normal", 9_999, 3, 2),               # odd d: general path, Philox blocks straddle buckets
    ("normal", 10_000, 4, 5),
    ("normal", 5_000, 1, 3),               # d = 1
    ("normal", 1, 512, 16),
    ("normal", 7, 512, 16),
    ("normal", 513, 512, 16),
    ("normal", 20_000, 512, 1 << 22),      # largest s
    ("normal", 20_000, 100, 7),            # d < 128: general
    # d not a multiple of 64, a large bucket with s > 31, sparse buckets
    ("normal", 100_000, 132, 3),
    ("normal", 200_000, 2048, 64),
    ("heavy_tailed_sparse", 300_000, 512, 2),
]


@pytest.mark.parametrize("kind,n,d,s", CASES, ids=["%s-n%d-d%d-s%d" % c for c in CASES])
def test_parity(oracle_lib, kind, n, d, s):
    v = vec(kind, n, n % 97 + d)
    check_parity(oracle_lib, v, d, s, seed=12345)


@pytest.mark.parametrize("d", [512, 1000, 3, 8192])
def test_parity_misaligned_input(oracle_lib, d):
    v = vec("normal", 50_003, 5)
    check_parity(oracle_lib, v, d, 16, seed=3, misalign=1)


def test_parity_large_seed(oracle_lib):
    v = vec("normal", 40_000, 8)
    check_parity(oracle_lib, v, 512, 16, seed=0xDEADBEEF12345678)


def test_special_values(oracle_lib):
    n, d = 512 * 16, 512
    v = vec("normal", n, 4)
    v[0:512] = 0.0                           # zero bucket
    v[512 + 7] = np.inf                      # non-finite bucket
    v[1024 + 3] = np.nan                     # non-finite bucket
    v[1536:2048] = -0.0                      # negative zeros: zero norm
    v[2048:2560] = 1e-30                     # squares underflow fp32: rescaled norm
    v[2560:3072] *= 1e-20                    # squares in the subnormal range: rescaled norm
    v[3072:3584] = np.float32(3.0)           # equal magnitudes: every coordinate non-zero
    v[3584:4096] = 0.0
    v[3584] = 5.0                            # one-hot
    v[4096:4608] = 0.0
    v[4096] = 1e-37                          # s / norm overflows for large s: RANGE
    v[4608:5120] = 1e30                      # squares overflow fp32: rescaled norm
    v[5120:5632] = 3e38                      # the norm itself overflows: NONFINITE
    v[5632:6144] = -v[5632:6144]
    check_parity(oracle_lib, v, d, 1 << 20, seed=7)
    check_parity(oracle_lib, v, d, 16, seed=7)


def test_empty_vector():
    import torch
    from quantized_gradient_compression_b200 import binding as B

    x = torch.empty(0, dtype=torch.float32, device="cuda")
    enc = B.encode(x, 512, 16, 0)
    torch.cuda.synchronize()
    assert enc.offsets.cpu().tolist() == [0]


def test_deterministic_and_workspace_reuse(oracle_lib):
    # alternating paths and sizes through one workspace; same input, same bits
    import torch
    from gpu_common import gpu_encode, device_vector

    shapes = [(200_000, 512, 16), (50_000, 3, 4), (300_000, 512, 16), (65_536, 8192, 1),
              (200_000, 512, 16)]
    first = {}
    for rep in range(2):
        for n, d, s in shapes:
            v = vec("normal", n, 11)
            _, words, offsets, _ = gpu_encode(device_vector(v), d, s, 9)
            key = (n, d, s)
            if key in first:
                assert np.array_equal(first[key][0], words)
                assert np.array_equal(first[key][1], offsets)
            else:
                first[key] = (words, offsets)
    for (n, d, s), (words, offsets) in first.items():
        v = vec("normal", n, 11)
        check_parity(oracle_lib, v, d, s, seed=9)


def test_non_default_stream(oracle_lib):
    import torch

    st = torch.cuda.Stream()
    v = vec("layered", 400_000, 2)
    with torch.cuda.stream(st):
        check_parity(oracle_lib, v, 512, 16, seed=1)


def test_one_workspace_serves_every_encoder(oracle_lib):
    """Calls of the two-launch encoder (d = 512) and of the one-pass encoders (d = 3,
    d = 8192) alternate on the binding's one shared workspace: each leaves it ready
    for the next."""
    for n, d, s, seed in ((70_001, 512, 16, 1), (30_001, 3, 4, 2), (70_001, 512, 16, 3),
                          (50_000, 8192, 1, 4), (10_000, 128, 64, 5)):
        check_parity(oracle_lib, W.layered(n, seed), d, s, seed)


def test_compaction_tiles_on_both_paths(oracle_lib):
    """Tiles of 256 buckets at s = 48: full tiles hold about 16,920 staged words,
    more than the compaction gathers into shared memory, so they copy from the
    staging slots; tiles with zero buckets hold fewer and are gathered."""
    n = 6 * 256 * 512
    v = W.normal(n, 3)
    v[256 * 512:256 * 512 + 60 * 512] = 0.0
    v[3 * 256 * 512:3 * 256 * 512 + 128 * 512] = 0.0
    check_parity(oracle_lib, v, 512, 48, seed=1)

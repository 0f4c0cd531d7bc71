"""Seeded synthetic gradients with the shapes of the benchmark workloads.

This module holds no codec arithmetic: it only draws numpy arrays.  Both the
CUDA path and the CPU oracle take their inputs from here.

Workload shapes (parameter counts of ResNet-50 / ResNet-152 gradients are used
only as sizes; no model, weights or dataset is involved):

=====  =============================================================  ==========  =====
name   input                                                          bucket d    s
=====  =============================================================  ==========  =====
c1     n=65,536 i.i.d. N(0,1), data seed 0                            65,536      256
c2     n=25,557,032 in 54 segments (Dirichlet(1) lengths, seed 1),    512         16
       segment i ~ N(0, sigma_i^2), log10 sigma_i ~ U[-4, -1]
c3     n=60,192,808 Student-t(3) * 1e-3, 1% exact zeros, data seed 2  8,192       1
c4     16 x n=25,557,032 N(0, 1e-4), data seeds 100+j, Philox seed j   512         4
c5     n=2^30 N(0,1), data seed 5                                     512         1,4,16,256
=====  =============================================================  ==========  =====
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

N_RESNET50 = 25_557_032
N_RESNET152 = 60_192_808


@dataclass(frozen=True)
class Workload:
    name: str
    n: int
    d: int
    s: int
    seed: int  # Philox seed
    data_seed: int
    kind: str  # generator kind

    def generate(self) -> np.ndarray:
        return GENERATORS[self.kind](self.n, self.data_seed)


def normal(n: int, data_seed: int, sigma: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng(data_seed)
    v = rng.standard_normal(n, dtype=np.float32)
    if sigma != 1.0:
        v *= np.float32(sigma)
    return v


def layered(n: int, data_seed: int, segments: int = 54) -> np.ndarray:
    """Concatenation of `segments` Gaussian layers of random lengths and scales.

    Lengths: floor of n times the cumulative Dirichlet(1,...,1) proportions; the
    last segment takes the remainder.  Scales: log10(sigma) ~ U[-4, -1]."""
    rng = np.random.default_rng(data_seed)
    props = rng.dirichlet(np.ones(segments))
    cuts = np.floor(np.cumsum(props)[:-1] * n).astype(np.int64)
    bounds = np.concatenate([[0], cuts, [n]])
    sigmas = 10.0 ** rng.uniform(-4.0, -1.0, size=segments)
    v = np.empty(n, dtype=np.float32)
    for i in range(segments):
        a, b = int(bounds[i]), int(bounds[i + 1])
        if b > a:
            v[a:b] = rng.standard_normal(b - a, dtype=np.float32) * np.float32(sigmas[i])
    return v


def heavy_tailed_sparse(n: int, data_seed: int) -> np.ndarray:
    """Student-t with 3 degrees of freedom, scaled by 1e-3, with 1% exact zeros."""
    rng = np.random.default_rng(data_seed)
    v = (rng.standard_t(3.0, size=n) * 1e-3).astype(np.float32)
    v[rng.random(n) < 0.01] = 0.0
    return v


def small_normal(n: int, data_seed: int) -> np.ndarray:
    """N(0, 1e-4), i.e. sigma = 0.01."""
    return normal(n, data_seed, sigma=0.01)


GENERATORS = {
    "normal": normal,
    "layered": layered,
    "heavy_tailed_sparse": heavy_tailed_sparse,
    "small_normal": small_normal,
}

C1 = Workload("c1_single_bucket_n65536", 65_536, 65_536, 256, 0, 0, "normal")
C2 = Workload("c2_resnet50_grad_d512_s16", N_RESNET50, 512, 16, 0, 1, "layered")
C3 = Workload("c3_resnet152_grad_d8192_s1", N_RESNET152, 8192, 1, 0, 2, "heavy_tailed_sparse")


def c4_streams(n: int = N_RESNET50, K: int = 16):
    """The K sender workloads of the receiver-aggregation case."""
    return [Workload("c4_sender%d" % j, n, 512, 4, j, 100 + j, "small_normal") for j in range(K)]


def c5(s: int, n: int = 1 << 30) -> Workload:
    return Workload("c5_n%d_d512_s%d" % (n, s), n, 512, s, 0, 5, "normal")


def scaled(w: Workload, n: int) -> Workload:
    """The same recipe at a smaller n (parity tests the oracle finishes quickly)."""
    return Workload(w.name + "_n%d" % n, n, w.d, w.s, w.seed, w.data_seed, w.kind)

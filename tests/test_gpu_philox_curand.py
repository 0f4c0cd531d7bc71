"""Pins the oracle's Philox counter/key layout against curand's Philox4_32_10
generator, run on the GPU (its source is not read).  This is the only pin of the
seed -> key mapping for seeds of 2^32 and above."""

import ctypes
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cuda", "philox_curand_probe.cu")
LIB = os.path.join(HERE, "cuda", "libphilox_curand_probe.so")


def _lib():
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                        "-Xcompiler", "-fPIC", SRC, "-o", LIB], check=True)
    return ctypes.CDLL(LIB)


def test_oracle_random_words_match_curand(oracle_lib):
    import torch

    seeds = [0, 1, 7, 0xFFFFFFFF, 1 << 32, 0x0123456789ABCDEF, 0xFFFFFFFFFFFFFFFF, 42 << 40]
    js = [0, 1, 2, 1000, (1 << 32) - 1, 1 << 32, 123456789012]
    pairs = [(s, j) for s in seeds for j in js]
    d_s = torch.from_numpy(np.array([p[0] for p in pairs], dtype=np.uint64)).cuda()
    d_j = torch.from_numpy(np.array([p[1] for p in pairs], dtype=np.uint64)).cuda()
    out = torch.zeros(4 * len(pairs), dtype=torch.int32, device="cuda")
    lib = _lib()
    rc = lib.philox_curand_probe(ctypes.c_void_p(d_s.data_ptr()), ctypes.c_void_p(d_j.data_ptr()),
                                 len(pairs), ctypes.c_void_p(out.data_ptr()))
    assert rc == 0
    got = out.cpu().numpy().view(np.uint32).reshape(-1, 4)
    for (seed, j), row in zip(pairs, got):
        expect = [oracle_lib.random_word(seed, 4 * j + w) for w in range(4)]
        assert [int(x) for x in row] == expect, (seed, j)

"""The data-parallel exchange on CPU: two and three gloo ranks.

The exchange's host logic (lengths, headers, padding, rank-major layout, per-rank
seeds, the order of the collectives) is the same for every codec.  These tests give it
a codec backed by the oracle on CPU tensors.  Every rank then checks its mean against
the oracle's mean of all ranks' streams, which it rebuilds locally from the seeded
gradients.  The CUDA codec takes the same path on the GPU (tests/test_gpu_exchange.py)."""

import json
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N, D, S, BW = 20_011, 256, 8, 4


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleCodec:
    """Elias streams from the oracle, held in CPU tensors laid out like the library's."""

    def __init__(self, o, n, d, s):
        import torch

        self.o, self.n, self.d, self.s = o, n, d, s
        self.nb = (n + d - 1) // d
        self.cap = o.capacity_words(n, d, s)
        self.words = torch.zeros(self.cap, dtype=torch.int32)
        self.offsets = torch.zeros(self.nb + 1, dtype=torch.int64)

    def encode(self, grad, memory, seed):
        import torch

        g = grad.numpy()
        if memory is None:
            w, off, _, _ = self.o.encode(g, self.d, self.s, seed)
        else:
            w, off, _, _, e_new = self.o.encode_ef(g, memory.numpy(), self.d, self.s, seed)
            memory.copy_(torch.from_numpy(e_new))
        self.words.zero_()
        self.words[: w.size] = torch.from_numpy(w.view(np.int32))
        self.offsets.copy_(torch.from_numpy(off.view(np.int64)))
        return self.words, self.offsets

    def stream_bits(self, offsets):
        return offsets[self.nb:self.nb + 1]

    def decode_mean(self, words, num_words, offsets, K, out):
        import torch

        wv = words.numpy().view(np.uint32)
        ov = offsets.numpy().view(np.uint64)
        streams = [(wv[j * num_words:(j + 1) * num_words], ov[j * (self.nb + 1):(j + 1) * (self.nb + 1)])
                   for j in range(K)]
        m, st = self.o.decode_mean(streams, self.n, self.d, self.s)
        assert st == 0
        out.copy_(torch.from_numpy(m))
        return out


class OracleBbitCodec:
    def __init__(self, o, n, d, b):
        import torch

        self.o, self.n, self.d, self.b = o, n, d, b
        self.nb = (n + d - 1) // d
        self.norms = torch.zeros(self.nb, dtype=torch.float32)
        self.codes = torch.zeros(o.bbit_code_words(n, b), dtype=torch.int32)

    def encode(self, grad, memory, seed):
        import torch

        if memory is None:
            c, nr, _ = self.o.bbit_encode(grad.numpy(), self.d, self.b, seed)
        else:
            c, nr, _, e_new = self.o.bbit_encode_ef(grad.numpy(), memory.numpy(), self.d, self.b, seed)
            memory.copy_(torch.from_numpy(e_new))
        self.norms.copy_(torch.from_numpy(nr))
        self.codes.copy_(torch.from_numpy(c.view(np.int32)))
        return self.norms, self.codes

    def decode_mean(self, norms, codes, K, out):
        import torch

        nv, cv = norms.numpy(), codes.numpy().view(np.uint32)
        m_n, m_c = self.nb, self.codes.numel()
        streams = [(nv[j * m_n:(j + 1) * m_n], cv[j * m_c:(j + 1) * m_c]) for j in range(K)]
        m, st = self.o.bbit_decode_mean(streams, self.n, self.d, self.b)
        assert st == 0
        out.copy_(torch.from_numpy(m))
        return out


def _grad(rank, step):
    from quantized_gradient_compression_b200 import workloads as W

    # ranks get gradients of very different sizes, so their streams differ in length
    return W.layered(N, 1000 * step + rank) * np.float32(10.0 ** rank)


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import oracle
    from quantized_gradient_compression_b200 import exchange as X

    o = oracle.default()
    res = {"ok": [], "max_words": []}
    # Elias, plain then with the error-feedback memory over three steps
    xe = X.EliasExchange(OracleCodec(o, N, D, S))
    for step in range(2):
        out = xe.step(torch.from_numpy(_grad(rank, step)), seed=7 + step)
        streams = []
        for j in range(world):
            w, off, _, _ = o.encode(_grad(j, step), D, S, X.rank_seed(7 + step, j))
            streams.append((w, off))
        ref, _ = o.decode_mean(streams, N, D, S)
        res["ok"].append(bool(np.array_equal(out.numpy().view(np.uint32), ref.view(np.uint32))))
        res["max_words"].append([xe.last.max_words, max((int(off[-1]) + 31) // 32 for _, off in streams)])
    mem = torch.zeros(N, dtype=torch.float32)
    mems = [np.zeros(N, np.float32) for _ in range(world)]
    for step in range(3):
        out = xe.step(torch.from_numpy(_grad(rank, step)), seed=50 + step, memory=mem)
        streams = []
        for j in range(world):
            w, off, _, _, mems[j] = o.encode_ef(_grad(j, step), mems[j], D, S, X.rank_seed(50 + step, j))
            streams.append((w, off))
        ref, _ = o.decode_mean(streams, N, D, S)
        res["ok"].append(bool(np.array_equal(out.numpy().view(np.uint32), ref.view(np.uint32))))
        res["ok"].append(bool(np.array_equal(mem.numpy().view(np.uint32), mems[rank].view(np.uint32))))
    # b-bit
    xb = X.BbitExchange(OracleBbitCodec(o, N, D, BW))
    out = xb.step(torch.from_numpy(_grad(rank, 0)), seed=3)
    streams = []
    for j in range(world):
        c, nr, _ = o.bbit_encode(_grad(j, 0), D, BW, X.rank_seed(3, j))
        streams.append((nr, c))
    ref, _ = o.bbit_decode_mean(streams, N, D, BW)
    res["ok"].append(bool(np.array_equal(out.numpy().view(np.uint32), ref.view(np.uint32))))
    # b-bit with the memory, two steps
    bmem = torch.zeros(N, dtype=torch.float32)
    bmems = [np.zeros(N, np.float32) for _ in range(world)]
    for step in range(2):
        out = xb.step(torch.from_numpy(_grad(rank, step)), seed=80 + step, memory=bmem)
        streams = []
        for j in range(world):
            c, nr, _, bmems[j] = o.bbit_encode_ef(_grad(j, step), bmems[j], D, BW, X.rank_seed(80 + step, j))
            streams.append((nr, c))
        ref, _ = o.bbit_decode_mean(streams, N, D, BW)
        res["ok"].append(bool(np.array_equal(out.numpy().view(np.uint32), ref.view(np.uint32))))
        res["ok"].append(bool(np.array_equal(bmem.numpy().view(np.uint32), bmems[rank].view(np.uint32))))
    # uneven streams: rank 0 sends an all-zero gradient (norms only), the others a
    # gradient with a non-finite bucket
    def odd(j):
        g = np.zeros(N, np.float32) if j == 0 else _grad(j, 9)
        if j > 0:
            g[D + 3] = np.inf
        return g
    out = xe.step(torch.from_numpy(odd(rank)), seed=99)
    streams = []
    for j in range(world):
        w, off, _, _ = o.encode(odd(j), D, S, X.rank_seed(99, j))
        streams.append((w, off))
    ref, _ = o.decode_mean(streams, N, D, S)
    res["ok"].append(bool(np.array_equal(out.numpy().view(np.uint32), ref.view(np.uint32))))
    res["mean0"] = float(out[0])
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_on_gloo_ranks(tmp_path, world):
    import torch.multiprocessing as mp

    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(world)]
    for i in range(world):
        assert all(r[i]["ok"]), (i, r[i]["ok"])
        for got, want in r[i]["max_words"]:
            assert got == want  # the payload is padded to the longest stream, not to capacity
    assert len({x["mean0"] for x in r}) == 1  # every rank holds the same mean


def test_rank_seeds_differ():
    from quantized_gradient_compression_b200 import exchange as X

    assert len({X.rank_seed(5, r) for r in range(8)}) == 8
    assert X.rank_seed(2**64 - 1, 1) == 0

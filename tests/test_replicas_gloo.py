"""The multi-process (replica) harness of bench.py on CPU: two gloo ranks.

The codec does not shard: under torchrun every rank runs an independent replica,
timed as the maximum over ranks, and the reference arm runs on rank 0 alone.  These
checks run the same helpers bench.py uses, with the gloo backend, no GPU."""

import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from quantized_gradient_compression_b200 import workloads as W

    t_mine = [1.5, 2.5][rank]
    res = {"max": bench.max_over_ranks(t_mine, world), "seed": bench.replica_seed(W.C2, rank),
           "value": bench.job_value(world, 4.0 * W.C2.n, bench.max_over_ranks(t_mine, world))}
    bench.barrier(world)
    # the reference arm: rank 0 alone runs it; here only the other rank calls it
    if rank == 1:
        class A:
            steps, warmup, gpus = 1, 3, world

        buf = io.StringIO()
        with redirect_stdout(buf):
            ret = bench.run_reference(A, W.C2)
        res["ref_output"] = buf.getvalue()
        res["ref_ret"] = ret
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
        json.dump(res, f)


def test_two_gloo_replicas(tmp_path):
    import torch.multiprocessing as mp

    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(world)]
    assert r[0]["max"] == r[1]["max"] == 2.5            # the slowest rank's time
    assert r[0]["seed"] != r[1]["seed"]                 # independent rounding per replica
    n = 25_557_032
    assert r[0]["value"] == pytest.approx(2 * 4.0 * n / 2.5 / 1e6)  # all ranks' bytes / max time
    assert r[1]["ref_output"] == "" and r[1]["ref_ret"] is None     # non-zero ranks do no work


def test_phase_spread():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.spread([3.0, 1.0, 2.0, 10.0]) == {"ms_median": 2.5, "ms_min": 1.0}
    assert bench.spread([0.5]) == {"ms_median": 0.5, "ms_min": 0.5}

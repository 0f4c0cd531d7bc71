"""QSGD codec benchmark on B200: encode, decode and decode-accumulate throughput.

One step is the whole hot path over one synthetic ResNet-50-sized gradient
(n = 25,557,032 fp32 in 54 Gaussian layers, bucket d = 512, s = 16):
  qsgd_encode (bucket norm, Philox stochastic rounding, Elias-omega packing,
  look-back scan) -> qsgd_decode (dense fp32) -> qsgd_decode_accumulate (the
  step's stream summed into a receiver buffer).
The metric is GB/s of fp32 gradient input (4n bytes per step) and the fraction of
the measured HBM roofline.  The L2 (126 MB, larger than the 110 MB working set of
a step) is flushed before every timed step by writing a 512 MB buffer.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs an independent replica (the codec does not
shard); the step time is the maximum over ranks and `value` counts all ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QSGD encode & decode GB/s of fp32 gradient input; % of B200 HBM roofline"
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic per call of each phase (dram__bytes_read.sum + dram__bytes_write.sum,
# summed over the call's launches: the encode's coder and compaction) from one ncu
# capture of this workload (ncu --set full over bench.py --profile-step), with the
# hash of the kernel sources it was taken on; reported as null once the sources
# differ.
TRAFFIC_SOURCES = ("qsgd_encode_stage.cu", "qsgd_decode_rows.cu", "qsgd_tables.cuh", "qsgd_device.cuh", "qsgd_limits.h")
TRAFFIC = {"bytes_per_launch": {"encode": 121090560, "decode": 51003648, "decode_accumulate": 153872896},
           "sources_sha256": "ed35e11c89e53d065d17348bdfa3b1047d226909ee6bfac3b3e850d810e0eb60"}


# The kernels behind each phase of the c2 step (d = 512, s = 16, aligned buffers).
KERNELS = {"encode": "code_buckets_short<4, false> + compact_stream (qsgd_encode, two launches)",
           "decode": "decode_rows<4, false> (qsgd_decode)",
           "decode_accumulate": "decode_rows<4, true> (qsgd_decode_accumulate, K = 1)"}


def sources_sha256() -> str:
    """Hash of the files that hold the device code of the profiled kernels (the
    bucket coder, the compaction and the row decoder): the traffic figures above are
    void once it changes."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_gradient_compression_b200", "csrc")
    for name in TRAFFIC_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5],
                    help="workload: 2 (default, the headline line) or another of the five configs")
    ap.add_argument("--profile-step", action="store_true",
                    help="no timing: run the config's step three times (two as warm-up) and exit, for a "
                         "profiler's capture of the third; c2 / c5 take --s")
    ap.add_argument("--s", type=int, default=None, help="levels for --profile-step on c2 or c5")
    ap.add_argument("--d", type=int, default=None,
                    help="bucket size for --profile-step on c2 (d % 4 != 0 takes the general encoder and the "
                         "any-shape decoder)")
    ap.add_argument("--bbit", type=int, default=None, choices=[2, 4, 8],
                    help="--profile-step on c2 with the fixed-width b-bit codec instead")
    return ap.parse_args()


def profile_step(args):
    """Three passes of one config's device work, untimed: c1 / c2 / c3 / c5 (at --s)
    qsgd_encode, qsgd_decode and qsgd_decode_accumulate (K = 1); c4 the sixteen
    senders' encodes and the K = 16 qsgd_decode_accumulate; with --bbit, the b-bit
    encode, decode and decode-accumulate on c2.  Launches per pass: two for each
    encode on the two-launch shapes, two for the decode of buckets past 1024
    coordinates (a fill, then the records), one for every other decode."""
    import torch
    from quantized_gradient_compression_b200 import binding as B
    from quantized_gradient_compression_b200 import workloads as W

    cfg = args.config
    if args.bbit is not None:
        w = W.C2
        x = torch.from_numpy(w.generate()).cuda()
        acc = torch.zeros(w.n, dtype=torch.float32, device="cuda")
        for _ in range(3):
            enc = B.bbit_encode(x, w.d, args.bbit, w.seed)
            B.bbit_decode(enc)
            B.bbit_decode_accumulate([enc], acc)
        torch.cuda.synchronize()
        return
    if cfg == 4:
        senders = W.c4_streams()
        xs = [torch.from_numpy(w.generate()).cuda() for w in senders]
        acc = torch.zeros(senders[0].n, dtype=torch.float32, device="cuda")
        for _ in range(3):
            encs = [B.encode(x, w.d, w.s, w.seed) for x, w in zip(xs, senders)]
            B.decode_accumulate(encs, acc)
        torch.cuda.synchronize()
        return
    w = {1: W.C1, 2: W.C2, 3: W.C3, 5: W.c5(16)}[cfg]
    s = args.s if args.s is not None and cfg in (2, 5) else w.s
    d = args.d if args.d is not None and cfg == 2 else w.d
    x = torch.from_numpy(w.generate()).cuda()
    acc = torch.zeros(w.n, dtype=torch.float32, device="cuda")
    for _ in range(3):
        enc = B.encode(x, d, s, w.seed)
        out, st = B.decode(enc)
        B.decode_accumulate([enc], acc)
    torch.cuda.synchronize()
    if int(enc.status.item()) != 0 or int(st.item()) != 0:
        raise RuntimeError("device status %d / %d" % (int(enc.status.item()), int(st.item())))


def workload():
    from quantized_gradient_compression_b200 import workloads as W

    return W.C2


def config_dict(w, extra=None):
    c = {"workload": w.name, "n": w.n, "bucket_d": w.d, "s": w.s, "philox_seed": w.seed,
         "data": "54 Gaussian layers, Dirichlet(1) lengths, log10 sigma ~ U[-4,-1], data seed %d"
                 % w.data_seed,
         "step": "encode -> decode -> decode_accumulate(K=1)",
         "l2": "flushed before every timed step (512 MB write)"}
    if extra:
        c.update(extra)
    return c


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                             "hw": parts[5], "hw_thermal": parts[6], "sw_thermal": parts[7],
                             "sw_power": parts[8]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(load)}


# --------------------------------------------------------------------------
# distributed plumbing (replicas; timing only)
# --------------------------------------------------------------------------
def init_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    """The maximum of x over the ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(w, rank: int) -> int:
    """Each replica encodes with its own Philox seed (its own gradient's rounding)."""
    return w.seed + rank


def spread(times) -> dict:
    """Median and minimum of per-step device times (ms)."""
    return {"ms_median": statistics.median(times), "ms_min": min(times)}


def job_value(world: int, bytes_per_rank: float, ms_max: float) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank / ms_max / 1e6


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# --------------------------------------------------------------------------
# the oracle as the CPU baseline / reference arm
# --------------------------------------------------------------------------
def time_oracle(v: np.ndarray, w, min_seconds: float = 10.0, max_reps: int = 3):
    import oracle

    o = oracle.default()
    reps, total = 0, 0.0
    while reps < max_reps and (reps == 0 or total < min_seconds):
        t0 = time.perf_counter()
        words, offsets, _, _ = o.encode(v, w.d, w.s, w.seed)
        o.decode(words, offsets, v.size, w.d, w.s)
        acc = np.zeros(v.size, dtype=np.float32)
        o.decode_accumulate([(words, offsets)], v.size, w.d, w.s, acc)
        total += time.perf_counter() - t0
        reps += 1
    per_step = total / reps
    return {"value": 4.0 * v.size / per_step / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "full workload vector (n=%d), %d step(s) of encode+decode+decode_accumulate, "
                      "single-threaded C oracle" % (v.size, reps),
            "seconds_per_step": per_step}


def run_reference(args, w):
    """The reference arm: the oracle (single-threaded C) on the host, as it stands.

    Every step encodes, decodes and decode-accumulates a bounded sample of the
    workload, sized from a probe so that the K timed steps take about a minute."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    v = w.generate()
    import oracle

    o = oracle.default()

    def step(vs):
        words, offsets, _, _ = o.encode(vs, w.d, w.s, w.seed)
        o.decode(words, offsets, vs.size, w.d, w.s)
        acc = np.zeros(vs.size, dtype=np.float32)
        o.decode_accumulate([(words, offsets)], vs.size, w.d, w.s, acc)

    probe_n = min(w.n, 1 << 20)
    t0 = time.perf_counter()
    step(np.ascontiguousarray(v[:probe_n]))
    rate = probe_n / (time.perf_counter() - t0)  # coordinates per second
    K = max(1, args.steps)
    sample_n = int(min(w.n, max(w.d, 60.0 / K * rate)))
    sample_n -= sample_n % w.d if sample_n > w.d else 0
    vs = np.ascontiguousarray(v[:sample_n])
    for _ in range(args.warmup):
        step(vs)
    t0 = time.perf_counter()
    for _ in range(K):
        step(vs)
    per_step = (time.perf_counter() - t0) / K
    value = 4.0 * sample_n / per_step / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": K, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config_dict(w, {"sample_n": sample_n}),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": "first %d coordinates of the workload per step" % sample_n},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def run_ours(args, w):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    rank, world, local = init_dist(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    v_host = w.generate()
    n, d, s = w.n, w.d, w.s
    seed = replica_seed(w, rank)
    nb = B.qsgd_num_buckets(n, d)
    cap = B.qsgd_max_encoded_words(n, d, s)
    x = torch.from_numpy(v_host).to(dev)
    words = torch.empty(cap, dtype=torch.int32, device=dev)
    offsets = torch.empty(nb + 1, dtype=torch.int64, device=dev)
    out = torch.empty(n, dtype=torch.float32, device=dev)
    acc = torch.zeros(n, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws_bytes = B.qsgd_encode_workspace_bytes(n, d, s)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def check(code, what):
        if code != 0:
            raise RuntimeError("%s failed: %s" % (what, B.qsgd_error_string(code)))

    def encode():
        check(B.qsgd_encode(x.data_ptr(), n, d, s, seed, words.data_ptr(), cap, offsets.data_ptr(),
                            ws.data_ptr(), ws_bytes, status.data_ptr(), sh), "qsgd_encode")

    def decode():
        check(B.qsgd_decode(words.data_ptr(), cap, offsets.data_ptr(), n, d, s, out.data_ptr(),
                            status.data_ptr(), sh), "qsgd_decode")

    def accumulate():
        check(B.qsgd_decode_accumulate([words.data_ptr()], [cap], [offsets.data_ptr()], 1, n, d, s,
                                       acc.data_ptr(), status.data_ptr(), sh), "qsgd_decode_accumulate")

    for _ in range(args.warmup):
        flush.zero_()
        encode()
        decode()
        accumulate()
    torch.cuda.synchronize()
    st = int(status.item())
    if st != 0:
        raise RuntimeError("device status %d after warm-up" % st)
    total_bits = int(offsets[-1].item())
    comp_bytes = 4 * ((total_bits + 31) // 32) + 8 * (nb + 1)

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for k in range(K):
            flush.zero_()
            ev[k][0].record(stream)
            encode()
            ev[k][1].record(stream)
            decode()
            ev[k][2].record(stream)
            accumulate()
            ev[k][3].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    t_enc = sum(ev[k][0].elapsed_time(ev[k][1]) for k in range(K)) / K
    t_dec = sum(ev[k][1].elapsed_time(ev[k][2]) for k in range(K)) / K
    t_acc = sum(ev[k][2].elapsed_time(ev[k][3]) for k in range(K)) / K
    t_step = sum(ev[k][0].elapsed_time(ev[k][3]) for k in range(K)) / K
    per_step = {name: [ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(K)]
                for i, name in enumerate(("encode", "decode", "decode_accumulate"))}
    t_step_max = max_over_ranks(t_step, world)
    if int(status.item()) != 0:
        raise RuntimeError("device status %d in the timed region" % int(status.item()))

    # end to end through the C ABI with host buffers.  Every step copies its whole
    # input in from pinned host memory, runs the three calls and copies its whole
    # result out.  Steps are pipelined: step k+1's input copy (copy-in stream) and
    # step k-1's result copy (copy-out stream) overlap step k's kernels (compute
    # stream), with double-buffered device input and result.
    h_in = torch.from_numpy(v_host).pin_memory()
    h_out = [torch.empty(n, dtype=torch.float32).pin_memory() for _ in range(2)]
    xs = [x, torch.empty_like(x)]
    accs = [acc, torch.zeros_like(acc)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run_calls(xb, accb):
        check(B.qsgd_encode(xb.data_ptr(), n, d, s, seed, words.data_ptr(), cap, offsets.data_ptr(),
                            ws.data_ptr(), ws_bytes, status.data_ptr(), sh), "qsgd_encode")
        check(B.qsgd_decode(words.data_ptr(), cap, offsets.data_ptr(), n, d, s, out.data_ptr(),
                            status.data_ptr(), sh), "qsgd_decode")
        check(B.qsgd_decode_accumulate([words.data_ptr()], [cap], [offsets.data_ptr()], 1, n, d, s,
                                       accb.data_ptr(), status.data_ptr(), sh), "qsgd_decode_accumulate")

    def e2e_step(k):
        b = k & 1
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(ev_cmp[b])  # step k-2's encoder is done with xs[b]
            xs[b].copy_(h_in, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if k >= 2:
            stream.wait_event(ev_out[b])  # step k-2's result has left accs[b]
        run_calls(xs[b], accs[b])
        ev_cmp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            h_out[b].copy_(accs[b], non_blocking=True)
            ev_out[b].record(s_out)

    E = args.e2e_steps
    for k in range(2):
        e2e_step(k)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(2, E + 2):
        e2e_step(k)
    e1.record(s_out)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / E, world)
    if int(status.item()) != 0:
        raise RuntimeError("device status %d in the end-to-end run" % int(status.item()))

    def time_alone(fn):
        """Median device time (ms) of one call, L2 flushed before each."""
        for _ in range(3):
            fn()
        ts = []
        for _ in range(max(3, min(K, 50))):
            flush.zero_()
            e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e_a.record(stream)
            fn()
            e_b.record(stream)
            torch.cuda.synchronize()
            ts.append(e_a.elapsed_time(e_b))
        return statistics.median(ts)

    # fixed-width b-bit variant on the same vector: each call timed alone, L2 flushed
    bbit = {}
    for bw in (2, 4, 8):
        cw = B.qsgd_bbit_code_words(n, bw)
        norms_b = torch.empty(nb, dtype=torch.float32, device=dev)
        codes_b = torch.empty(max(cw, 1), dtype=torch.int32, device=dev)
        out_b = torch.empty(n, dtype=torch.float32, device=dev)
        acc_b = torch.zeros(n, dtype=torch.float32, device=dev)

        def b_enc():
            check(B.qsgd_bbit_encode(x.data_ptr(), n, d, bw, seed, norms_b.data_ptr(), codes_b.data_ptr(),
                                     status.data_ptr(), sh), "qsgd_bbit_encode")

        def b_dec():
            check(B.qsgd_bbit_decode(norms_b.data_ptr(), codes_b.data_ptr(), n, d, bw, out_b.data_ptr(),
                                     status.data_ptr(), sh), "qsgd_bbit_decode")

        def b_acc():
            check(B.qsgd_bbit_decode_accumulate([norms_b.data_ptr()], [codes_b.data_ptr()], 1, n, d, bw,
                                                acc_b.data_ptr(), status.data_ptr(), sh),
                  "qsgd_bbit_decode_accumulate")

        times = {name: time_alone(fn) for name, fn in
                 (("encode", b_enc), ("decode", b_dec), ("decode_accumulate", b_acc))}
        if int(status.item()) != 0:
            raise RuntimeError("device status %d in the b-bit runs" % int(status.item()))
        cbytes = 4.0 * nb + 4.0 * cw
        alg = {"encode": 4.0 * n + cbytes, "decode": cbytes + 4.0 * n, "decode_accumulate": cbytes + 8.0 * n}
        bbit["b%d" % bw] = {
            "s": (1 << (bw - 1)) - 1, "bits_per_coord": bw + 32.0 * nb / n,
            "us": {k: 1e3 * v for k, v in times.items()},
            "algorithmic_gbs": {k: alg[k] / times[k] / 1e6 for k in times},
            "roofline_frac": {k: alg[k] / times[k] / 1e6 / measured_peaks()[0] for k in times},
        }

    # QSGDinf (max-norm scale) on the same vector, Elias coded at the same (d, s): the
    # encoder and decoder timed alone, L2 flushed
    def i_enc():
        check(B.qsgd_encode_ex(x.data_ptr(), n, d, s, seed, B.QSGD_NORM_MAX, words.data_ptr(), cap,
                               offsets.data_ptr(), ws.data_ptr(), ws_bytes, status.data_ptr(), sh), "qsgd_encode_ex")

    def i_dec():
        check(B.qsgd_decode(words.data_ptr(), cap, offsets.data_ptr(), n, d, s, out.data_ptr(),
                            status.data_ptr(), sh), "qsgd_decode")

    i_times = {"encode": time_alone(i_enc), "decode": time_alone(i_dec)}
    if int(status.item()) != 0:
        raise RuntimeError("device status %d in the max-norm runs" % int(status.item()))
    i_bits = int(offsets[-1].item())
    i_comp = 4 * ((i_bits + 31) // 32) + 8 * (nb + 1)
    i_alg = {"encode": 4.0 * n + i_comp, "decode": i_comp + 4.0 * n}
    qsgdinf = {"s": s, "bits_per_coord": i_bits / n, "compressed_bytes": i_comp,
               "us": {k: 1e3 * v for k, v in i_times.items()},
               "algorithmic_gbs": {k: i_alg[k] / i_times[k] / 1e6 for k in i_times},
               "roofline_frac": {k: i_alg[k] / i_times[k] / 1e6 / measured_peaks()[0] for k in i_times}}

    # error feedback on the same gradient: the fused one-pass encode that reads g and
    # the memory e and writes the stream and e (L2 scale), timed alone, L2 flushed
    e_mem = torch.zeros(n, dtype=torch.float32, device=dev)

    def f_enc():
        check(B.qsgd_encode_ef(x.data_ptr(), e_mem.data_ptr(), n, d, s, seed, B.QSGD_NORM_L2, words.data_ptr(), cap,
                               offsets.data_ptr(), ws.data_ptr(), ws_bytes, status.data_ptr(), sh), "qsgd_encode_ef")

    f_ms = time_alone(f_enc)
    if int(status.item()) != 0:
        raise RuntimeError("device status %d in the error-feedback runs" % int(status.item()))
    f_bits = int(offsets[-1].item())
    f_comp = 4 * ((f_bits + 31) // 32) + 8 * (nb + 1)
    f_alg = 12.0 * n + f_comp  # read g and e, write e and the stream
    error_feedback = {"s": s, "bits_per_coord": f_bits / n, "us": {"encode": 1e3 * f_ms},
                      "algorithmic_bytes": f_alg, "algorithmic_gbs": {"encode": f_alg / f_ms / 1e6},
                      "roofline_frac": {"encode": f_alg / f_ms / 1e6 / measured_peaks()[0]}}

    # data-parallel exchange, every rank: encode, all-gather the lengths, headers and
    # padded streams (NCCL), decode the mean of the N streams; timed per step on the
    # device, max over ranks.  And the receiver's side of an 8-GPU node on this GPU: the
    # mean of 8 streams (this rank's stream 8 times), timed alone.
    from quantized_gradient_compression_b200 import exchange as X

    xch = X.EliasExchange(X.LibraryCodec(n, d, s, dev))
    xout = torch.empty(n, dtype=torch.float32, device=dev)
    for k in range(3):
        xch.step(x, seed + 1000 + k, out=xout)
    x_ts = []
    for k in range(max(3, min(K, 20))):
        flush.zero_()
        barrier(world)
        e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_a.record(stream)
        xch.step(x, seed + 2000 + k, out=xout)
        e_b.record(stream)
        torch.cuda.synchronize()
        x_ts.append(e_a.elapsed_time(e_b))
    x_ms = max_over_ranks(statistics.median(x_ts), world)
    if int(xch.codec.status.item()) != 0:
        raise RuntimeError("device status %d in the exchange" % int(xch.codec.status.item()))
    R = 8
    xw, xo = xch.codec.words, xch.codec.offsets

    def r_mean():
        check(B.qsgd_decode_mean([xw.data_ptr()] * R, [xw.numel()] * R, [xo.data_ptr()] * R, R, n, d, s,
                                 xout.data_ptr(), status.data_ptr(), sh), "qsgd_decode_mean")

    r_ms = time_alone(r_mean)
    r_comp = 4 * ((int(xo[-1].item()) + 31) // 32) + 8 * (nb + 1)
    exchange = {"ranks": world, "collective": "all_gather_into_tensor x3 (%s)" % (
                    "nccl" if world > 1 else "nccl, one rank" if torch.distributed.is_initialized() else "none"),
                "ms_per_step": x_ms, "sent_bytes_per_rank": xch.last.sent_bytes,
                "receiver_mean_of_8": {"us": 1e3 * r_ms, "algorithmic_bytes": R * r_comp + 4.0 * n,
                                       "roofline_frac": (R * r_comp + 4.0 * n) / r_ms / 1e6 / measured_peaks()[0]}}

    peak, peak_kind = measured_peaks()
    in_bytes = 4.0 * n
    enc_bytes = in_bytes + comp_bytes            # read fp32, write stream + header
    dec_bytes = comp_bytes + in_bytes            # read stream + header, write fp32
    acc_bytes = comp_bytes + 2 * in_bytes        # read stream, read + write the sum
    phases = {
        "encode": {"ms": t_enc, "input_gbs": in_bytes / t_enc / 1e6,
                   "algorithmic_gbs": enc_bytes / t_enc / 1e6, "roofline_frac": enc_bytes / t_enc / 1e6 / peak},
        "decode": {"ms": t_dec, "input_gbs": in_bytes / t_dec / 1e6,
                   "algorithmic_gbs": dec_bytes / t_dec / 1e6, "roofline_frac": dec_bytes / t_dec / 1e6 / peak},
        "decode_accumulate": {"ms": t_acc, "input_gbs": in_bytes / t_acc / 1e6,
                              "algorithmic_gbs": acc_bytes / t_acc / 1e6,
                              "roofline_frac": acc_bytes / t_acc / 1e6 / peak},
    }
    for name, ts in per_step.items():
        phases[name].update(spread(ts))  # "ms" is the mean over the timed steps
    dominant = max(phases, key=lambda k: phases[k]["ms"])
    dom = phases[dominant]
    traffic = None
    if TRAFFIC["sources_sha256"] == sources_sha256():
        traffic = TRAFFIC["bytes_per_launch"][dominant]

    result = {
        "metric": METRIC,
        "value": job_value(world, in_bytes, t_step_max),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": t_step_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": config_dict(w, {"parallelism": "replicas x%d" % world}),
        "bits_per_coord": total_bits / n,
        "compressed_bytes": comp_bytes,
        "phases": phases,
        "roofline": {"bound": "hbm", "kernel": KERNELS[dominant],
                     "achieved": dom["algorithmic_gbs"], "peak": peak, "unit": "GB/s",
                     "frac": dom["algorithmic_gbs"] / peak, "traffic": traffic,
                     "peak_source": "%s hbm_gbs (burst copy)" % peak_kind,
                     "algorithmic_bytes_per_launch": {"encode": enc_bytes, "decode": dec_bytes,
                                                      "decode_accumulate": acc_bytes}[dominant]},
        "e2e": {"value": job_value(world, in_bytes, t_e2e), "unit": "GB/s",
                "h2d_bytes_per_step": int(in_bytes), "d2h_bytes_per_step": int(in_bytes),
                "ms_per_step": t_e2e,
                "how": "qsgd_encode/decode/decode_accumulate on host-pinned data; per step H2D of the "
                       "input and D2H of the result, pipelined over copy-in / compute / copy-out streams"},
        "gpu_launches": 4 * K,  # per step: the encoder's coder and compaction, the decode, the accumulate
        "bbit": bbit,
        "qsgdinf": qsgdinf,
        "error_feedback": error_feedback,
        "exchange": exchange,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = time_oracle(v_host, w)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


# --------------------------------------------------------------------------
# the other configurations: one JSON line each (c2 above is the default line)
# --------------------------------------------------------------------------
CONFIG_NAMES = {1: "c1_single_bucket_n65536", 3: "c3_resnet152_grad_d8192_s1",
                4: "c4_receiver_K16_n25557032_d512_s4", 5: "c5_n1073741824_d512_s_sweep"}


def config_workloads(cfg: int):
    from quantized_gradient_compression_b200 import workloads as W

    if cfg == 1:
        return [W.C1]
    if cfg == 3:
        return [W.C3]
    if cfg == 4:
        return W.c4_streams()
    return [W.c5(s) for s in (1, 4, 16, 256)]


def run_config(args, cfg: int):
    """c1 / c3: encode and decode of one vector; c4: the 16 senders' encodes and the
    receiver's qsgd_decode_accumulate of all 16 streams; c5: encode and decode of the
    2^30 vector for s = 1, 4, 16, 256.  Every call is timed alone on the device (CUDA
    events, L2 flushed before each), median over the steps; value = GB/s of fp32
    gradient input of the config's step."""
    import torch
    from quantized_gradient_compression_b200 import binding as B

    rank, world, local = init_dist(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    peak, peak_kind = measured_peaks()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    K = args.steps

    def check(code, what):
        if code != 0:
            raise RuntimeError("%s failed: %s" % (what, B.qsgd_error_string(code)))

    def time_calls(fn):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(K):
            flush.zero_()
            e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e_a.record(stream)
            fn()
            e_b.record(stream)
            torch.cuda.synchronize()
            ts.append(e_a.elapsed_time(e_b))
        if int(status.item()) != 0:
            raise RuntimeError("device status %d" % int(status.item()))
        return statistics.median(ts), min(ts)

    ws_list = config_workloads(cfg)
    n, d = ws_list[0].n, ws_list[0].d
    nb = B.qsgd_num_buckets(n, d)
    lines = []
    with ClockSampler(local) as clocks:
        if cfg in (1, 3, 5):
            v_host = ws_list[0].generate()
            x = torch.from_numpy(v_host).to(dev)
            out = torch.empty(n, dtype=torch.float32, device=dev)
            for w in ws_list:
                s = w.s
                cap = B.qsgd_max_encoded_words(n, d, s)
                words = torch.empty(cap, dtype=torch.int32, device=dev)
                offsets = torch.empty(nb + 1, dtype=torch.int64, device=dev)
                ws_bytes = B.qsgd_encode_workspace_bytes(n, d, s)
                ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)

                def enc():
                    check(B.qsgd_encode(x.data_ptr(), n, d, s, replica_seed(w, rank), words.data_ptr(), cap,
                                        offsets.data_ptr(), ws.data_ptr(), ws_bytes, status.data_ptr(), sh),
                          "qsgd_encode")

                def dec():
                    check(B.qsgd_decode(words.data_ptr(), cap, offsets.data_ptr(), n, d, s, out.data_ptr(),
                                        status.data_ptr(), sh), "qsgd_decode")

                t_enc, m_enc = time_calls(enc)
                t_dec, m_dec = time_calls(dec)
                bits = int(offsets[-1].item())
                comp = 4 * ((bits + 31) // 32) + 8 * (nb + 1)
                alg = 4.0 * n + comp
                lines.append({"s": s, "bits_per_coord": bits / n, "compressed_bytes": comp,
                              "encode": {"ms_median": t_enc, "ms_min": m_enc, "input_gbs": 4.0 * n / t_enc / 1e6,
                                         "algorithmic_gbs": alg / t_enc / 1e6, "roofline_frac": alg / t_enc / 1e6 / peak},
                              "decode": {"ms_median": t_dec, "ms_min": m_dec, "input_gbs": 4.0 * n / t_dec / 1e6,
                                         "algorithmic_gbs": alg / t_dec / 1e6, "roofline_frac": alg / t_dec / 1e6 / peak}})
                del words, ws
            step_ms = sum(r["encode"]["ms_median"] + r["decode"]["ms_median"] for r in lines)
            value = len(lines) * 4.0 * n / step_ms / 1e6
            dom = max(((r["encode"]["ms_median"], "encode", r) for r in lines), key=lambda z: z[0])
            dom2 = max(((r["decode"]["ms_median"], "decode", r) for r in lines), key=lambda z: z[0])
            dom = max(dom, dom2, key=lambda z: z[0])
            roof = {"bound": "hbm", "kernel": "%s, s = %d" % (dom[1], dom[2]["s"]),
                    "achieved": dom[2][dom[1]]["algorithmic_gbs"], "peak": peak, "unit": "GB/s",
                    "frac": dom[2][dom[1]]["roofline_frac"], "traffic": None,
                    "peak_source": "%s hbm_gbs (burst copy)" % peak_kind}
            step = "encode -> decode" + (" for s = 1, 4, 16, 256" if cfg == 5 else "")
            extra = {"sweep": lines} if cfg == 5 else {"phases": {"encode": lines[0]["encode"], "decode": lines[0]["decode"]},
                                                       "bits_per_coord": lines[0]["bits_per_coord"],
                                                       "compressed_bytes": lines[0]["compressed_bytes"]}
            cpu_sample = v_host[: min(n, 1 << 22)]
            cpu_w = ws_list[2] if cfg == 5 else ws_list[0]
        else:  # c4: 16 senders, one receiver
            Kst = len(ws_list)
            s = ws_list[0].s
            cap = B.qsgd_max_encoded_words(n, d, s)
            ws_bytes = B.qsgd_encode_workspace_bytes(n, d, s)
            ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
            words = [torch.empty(cap, dtype=torch.int32, device=dev) for _ in range(Kst)]
            offsets = [torch.empty(nb + 1, dtype=torch.int64, device=dev) for _ in range(Kst)]
            xs = [torch.from_numpy(w.generate()).to(dev) for w in ws_list]
            acc = torch.zeros(n, dtype=torch.float32, device=dev)

            def enc_all():
                for j, w in enumerate(ws_list):
                    check(B.qsgd_encode(xs[j].data_ptr(), n, d, s, replica_seed(w, rank), words[j].data_ptr(), cap,
                                        offsets[j].data_ptr(), ws.data_ptr(), ws_bytes, status.data_ptr(), sh),
                          "qsgd_encode")

            def receive():
                check(B.qsgd_decode_accumulate([t.data_ptr() for t in words], [cap] * Kst,
                                               [t.data_ptr() for t in offsets], Kst, n, d, s, acc.data_ptr(),
                                               status.data_ptr(), sh), "qsgd_decode_accumulate")

            t_enc, m_enc = time_calls(enc_all)
            t_acc, m_acc = time_calls(receive)
            comps = []
            for o in offsets:
                bits = int(o[-1].item())
                comps.append(4 * ((bits + 31) // 32) + 8 * (nb + 1))
            alg_acc = sum(comps) + 8.0 * n
            alg_enc = Kst * 4.0 * n + sum(comps)
            value = Kst * 4.0 * n / t_acc / 1e6
            roof = {"bound": "hbm", "kernel": "qsgd_decode_accumulate, K = %d" % Kst,
                    "achieved": alg_acc / t_acc / 1e6, "peak": peak, "unit": "GB/s",
                    "frac": alg_acc / t_acc / 1e6 / peak, "traffic": None,
                    "peak_source": "%s hbm_gbs (burst copy)" % peak_kind}
            step = "decode_accumulate of the K = 16 streams into one fp32 buffer (the senders' encodes timed apart)"
            extra = {"bits_per_coord": sum(8 * c for c in comps) / Kst / n,
                     "phases": {"decode_accumulate_K16": {"ms_median": t_acc, "ms_min": m_acc,
                                                          "algorithmic_bytes": alg_acc,
                                                          "algorithmic_gbs": alg_acc / t_acc / 1e6,
                                                          "roofline_frac": alg_acc / t_acc / 1e6 / peak},
                                "encode_16_senders": {"ms_median": t_enc, "ms_min": m_enc,
                                                      "algorithmic_bytes": alg_enc,
                                                      "algorithmic_gbs": alg_enc / t_enc / 1e6,
                                                      "roofline_frac": alg_enc / t_enc / 1e6 / peak}}}
            step_ms = t_acc
            cpu_sample = ws_list[0].generate()[: 1 << 22]
            cpu_w = ws_list[0]
    # library launches per timed step: an encode is two (the coder and the compaction,
    # or the descriptor clear and the one-pass encoder), a decode one, the K = 16
    # receive one
    launches = K * (1 if cfg == 4 else 3 * len(ws_list))
    result = {"metric": METRIC, "value": world * value,
              "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms,
              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
              "config": {"workload": CONFIG_NAMES[cfg], "n": n, "bucket_d": d,
                         "s": [w.s for w in ws_list] if cfg == 5 else ws_list[0].s,
                         "step": step, "l2": "flushed before every timed call (512 MB write)",
                         "parallelism": "replicas x%d" % world},
              "roofline": roof, "gpu_launches": launches, "clocks": clocks.summary()}
    result.update(extra)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        o = oracle.default()
        t0 = time.perf_counter()
        reps = 0
        while reps < 3 and (reps == 0 or time.perf_counter() - t0 < 10.0):
            wds, offs, _, _ = o.encode(cpu_sample, cpu_w.d, cpu_w.s, cpu_w.seed)
            o.decode(wds, offs, cpu_sample.size, cpu_w.d, cpu_w.s)
            reps += 1
        per = (time.perf_counter() - t0) / reps
        result["cpu_baseline"] = {"value": 4.0 * cpu_sample.size / per / 1e9, "unit": "GB/s", "cores": 1,
                                  "kind": "oracle",
                                  "sample": "first %d coordinates, encode + decode at s = %d, single-threaded C oracle"
                                            % (cpu_sample.size, cpu_w.s)}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def main():
    args = parse_args()
    w = workload()
    if args.profile_step:
        profile_step(args)
        return
    if args.impl == "reference":
        if args.config != 2:
            w = config_workloads(args.config)[2 if args.config == 5 else 0]
        run_reference(args, w)
    elif args.config != 2:
        run_config(args, args.config)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()

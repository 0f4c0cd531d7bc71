"""The decoders' kernel source run on the CPU under a warp emulator (no GPU).

`tests/emu/inc/warp_emu.h` stands in for the CUDA features `decode_multi` (P = -1
below) and `decode_warp` (P = -2) use: every thread of a block is a host thread, and
each warp primitive gathers the 32 lanes and checks that they call the same primitive
at the same source line.  A lane that skips a primitive the others wait in (a
deadlock on a GPU) fails the test here, as does any mismatch with the oracle.
Shared memory starts as garbage, as on the device.  The kernel text is taken from
`qsgd_decode.cu` as it stands; only the launch helpers are cut.

The streams are made by the oracle; the checks are bit-exact.
"""

import os
import re
import shutil
import subprocess

import numpy as np
import pytest

from quantized_gradient_compression_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_gradient_compression_b200", "csrc")


def _kernel_source() -> str:
    src = open(os.path.join(CSRC, "qsgd_decode.cu")).read()
    # everything from the first host-side launch helper on is cut
    cut = src.index("cudaError_t launch_multi(const DecodeArgs& a, cudaStream_t stream) {")
    s = src[:cut] + "}  // namespace\n}  // namespace qsgd\n"
    s = s.replace('#include "../../include/qsgd.h"', '#include "%s"' % os.path.join(ROOT, "include", "qsgd.h"))
    s = s.replace('#include "qsgd_internal.h"', '#include "%s"' % os.path.join(CSRC, "qsgd_internal.h"))
    s = s.replace('#include "qsgd_tables.cuh"', '#include "%s"' % os.path.join(CSRC, "qsgd_tables.cuh"))
    s = s.replace("extern __shared__ __align__(16) uint32_t smem[];",
                  "uint32_t* smem = reinterpret_cast<uint32_t*>(g_emu_smem);")
    assert "asm" not in s
    return s


@pytest.fixture(scope="module")
def emu_exe(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("emu")
    with open(d / "decode_emu.inc", "w") as f:
        f.write(_kernel_source())
    exe = d / "emu_main"
    r = subprocess.run(["g++", "-O1", "-std=c++17", "-ffp-contract=off", "-pthread",
                        "-I", os.path.join(HERE, "emu", "inc"), "-I", str(d),
                        os.path.join(HERE, "emu", "emu_main.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    return str(exe)


def _flip_bits(words, offsets, rng):
    nb = offsets.size - 1
    for b in rng.integers(0, nb, size=max(1, nb // 8)):
        lo, hi = int(offsets[b]) + 32, int(offsets[b + 1])
        if hi > lo:
            for pos in rng.integers(lo, hi, size=3):
                words[pos >> 5] ^= np.uint32(1) << np.uint32(31 - (pos & 31))


def _run(exe, tmp, oracle_lib, n, d, s, K, P, accumulate, kind, corrupt=False, mean=False):
    streams = []
    for j in range(K):
        v = W.GENERATORS[kind](n, 300 + j)
        words, offsets, _, st = oracle_lib.encode(v, d, s, seed=77 + j)
        assert st == 0
        if corrupt:
            _flip_bits(words, offsets, np.random.default_rng(j))
        streams.append((words, offsets))
        np.concatenate([words, np.zeros(1, np.uint32)]).tofile(tmp / ("w%d.bin" % j))
        offsets.astype(np.uint64).tofile(tmp / ("o%d.bin" % j))
    base = (np.random.default_rng(d).standard_normal(n) * 1e-3).astype(np.float32)
    base[::5] = np.float32(-0.0)
    if not accumulate:
        base[:] = np.float32(np.nan)  # every coordinate must be written
    base.tofile(tmp / "out_in.bin")
    np.array([n, d, s, K], np.uint64).tofile(tmp / "params.bin")
    r = subprocess.run([exe, str(tmp), str(P), "1" if accumulate else "0", "3", "1" if mean else "0"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, (r.stdout[-500:], r.stderr[-2000:])
    status = int(r.stdout.split()[-1])
    got = np.fromfile(tmp / "out.bin", np.float32)
    return got, status, streams, base


# (n, d, s, K, P, accumulate, input): P = -2, the any-shape decoder (decode_warp),
# on the shapes the row decoders take on the GPU: ragged last group, d % 64 != 0,
# several streams in one launch
CASES = [
    (30_001, 512, 16, 1, -2, False, "layered"),
    (30_001, 512, 16, 2, -2, True, "layered"),
    (20_000, 100, 7, 2, -2, True, "normal"),
    (9_000, 132, 3, 1, -2, False, "normal"),
    (20_000, 512, 2, 1, -2, False, "heavy_tailed_sparse"),
    (9_001, 4096, 1000, 1, -2, False, "normal"),
    (513, 512, 16, 2, -2, True, "normal"),
]


@pytest.mark.parametrize("n,d,s,K,P,accumulate,kind", CASES,
                         ids=["n%d-d%d-s%d-K%d-P%d-%s-%s" % c for c in CASES])
def test_staged_decoder_matches_oracle(emu_exe, tmp_path, oracle_lib, n, d, s, K, P, accumulate, kind):
    got, status, streams, base = _run(emu_exe, tmp_path, oracle_lib, n, d, s, K, P, accumulate, kind)
    assert status == 0
    if accumulate:
        ref = base.copy()
        _, rst = oracle_lib.decode_accumulate(streams, n, d, s, ref)
    else:
        ref, rst = oracle_lib.decode(streams[-1][0], streams[-1][1], n, d, s)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("d", [512, 132, 2048])
def test_staged_decoder_corrupt_streams(emu_exe, tmp_path, oracle_lib, d):
    """Bit flips in some buckets: the kernel finishes (no lane waits alone), flags
    the stream, and every bucket without a flip decodes as the oracle decodes it."""
    n, s = 30_000, 16
    got, status, streams, _ = _run(emu_exe, tmp_path, oracle_lib, n, d, s, 1, -2, False, "normal", corrupt=True)
    assert status & 2
    words, offsets, _, _ = oracle_lib.encode(W.GENERATORS["normal"](n, 300), d, s, seed=77)
    ref, _ = oracle_lib.decode(words, offsets, n, d, s)
    flipped = streams[0][0] != words
    keep = np.ones(n, dtype=bool)
    for b in range(offsets.size - 1):
        w0, w1 = int(offsets[b]) >> 5, (int(offsets[b + 1]) + 31) >> 5
        if flipped[w0:w1].any():
            keep[b * d:min(n, (b + 1) * d)] = False
    assert keep.any()
    assert np.array_equal(got[keep].view(np.uint32), ref[keep].view(np.uint32))


# decode_multi (P = -1): K streams side by side in one launch (16 to a launch), for
# decode-accumulate and for the mean; ragged tails, d % 64 != 0, K past one chunk of
# eight warps and past one launch
MULTI = [
    # one, two, three and four streams: 8, 4, 2 and 2 groups to a CTA (3 leaves two
    # warps idle); bucket counts that leave the last set of groups part-filled
    (20_000, 512, 16, 1, True, False, "layered"),
    (70_001, 256, 16, 2, True, False, "normal"),
    (50_000, 100, 7, 4, True, False, "normal"),
    (33_000, 128, 5, 1, False, True, "normal"),
    (61_001, 256, 16, 2, False, True, "layered"),
    (20_000, 512, 16, 3, True, False, "layered"),
    (20_000, 512, 16, 8, True, False, "normal"),
    (9_001, 100, 7, 11, True, False, "normal"),
    (5_000, 132, 3, 17, True, False, "normal"),
    (20_000, 512, 16, 5, False, True, "layered"),
    (7_000, 100, 7, 18, False, True, "normal"),
    (4_000, 512, 16, 1, False, True, "normal"),
]


@pytest.mark.parametrize("n,d,s,K,accumulate,mean,kind", MULTI, ids=["n%d-d%d-s%d-K%d-acc%d-mean%d-%s" % c for c in MULTI])
def test_multi_stream_kernel_matches_oracle(emu_exe, tmp_path, oracle_lib, n, d, s, K, accumulate, mean, kind):
    got, status, streams, base = _run(emu_exe, tmp_path, oracle_lib, n, d, s, K, -1, accumulate, kind, mean=mean)
    assert status == 0
    if mean:
        ref, rst = oracle_lib.decode_mean(streams, n, d, s)
    else:
        ref = base.copy()
        _, rst = oracle_lib.decode_accumulate(streams, n, d, s, ref)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_multi_stream_kernel_corrupt_stream(emu_exe, tmp_path, oracle_lib):
    """Bit flips in stream 1 of 3: the kernel finishes, flags the input, and every
    bucket that no flip touched equals the oracle's sum."""
    n, d, s = 20_000, 512, 16
    got, status, streams, base = _run(emu_exe, tmp_path, oracle_lib, n, d, s, 3, -1, True, "normal", corrupt=True)
    assert status & 2
    intact = []
    for j in range(3):
        words, offsets, _, _ = oracle_lib.encode(W.GENERATORS["normal"](n, 300 + j), d, s, seed=77 + j)
        intact.append((words, offsets))
    ref = base.copy()
    oracle_lib.decode_accumulate(intact, n, d, s, ref)
    keep = np.ones(n, dtype=bool)
    for j in range(3):
        flipped = streams[j][0] != intact[j][0]
        offs = intact[j][1]
        for b in range(offs.size - 1):
            w0, w1 = int(offs[b]) >> 5, (int(offs[b + 1]) + 31) >> 5
            if flipped[w0:w1].any():
                keep[b * d:min(n, (b + 1) * d)] = False
    assert keep.any()
    assert np.array_equal(got[keep].view(np.uint32), ref[keep].view(np.uint32))


# decode_warp (P = -2): the decoder of every other shape (d % 4 != 0, d > 4096,
# s >= 1024), up to 16 streams to a launch with per-lane state in shared memory
WARP = [
    (20_000, 100, 7, 1, False, "normal"),
    (20_001, 130, 3, 3, True, "layered"),
    (9_001, 5_000, 2_000, 1, False, "normal"),
    (6_000, 99, 16, 17, True, "normal"),
    (30_000, 512, 16, 2, True, "heavy_tailed_sparse"),
]


@pytest.mark.parametrize("n,d,s,K,accumulate,kind", WARP, ids=["n%d-d%d-s%d-K%d-acc%d-%s" % c for c in WARP])
def test_general_decoder_matches_oracle(emu_exe, tmp_path, oracle_lib, n, d, s, K, accumulate, kind):
    got, status, streams, base = _run(emu_exe, tmp_path, oracle_lib, n, d, s, K, -2, accumulate, kind)
    assert status == 0
    if accumulate:
        ref = base.copy()
        _, rst = oracle_lib.decode_accumulate(streams, n, d, s, ref)
    else:
        ref, rst = oracle_lib.decode(streams[-1][0], streams[-1][1], n, d, s)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))

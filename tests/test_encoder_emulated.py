"""The encoder kernels' exact source on a CPU warp and block emulator (no GPU).

`encode_fast` (with and without the error-feedback memory) and `encode_general` are
compiled for the host under tests/emu/enc/block_emu.h.  The whole grid runs at once:
every CUDA thread is a host thread, and the CTAs hand tiles to one another as on the
device.  Each warp primitive checks that its 32 lanes meet at the same call site.
The stream and offsets are compared bit for bit with the oracle's encode under the
emulated encoder's own norms (the wire format lets an encoder choose its fp32 norm
within 1e-6); the memory with the oracle's error-feedback encode."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from emu_source import host_source as _host_source
from gpu_common import check_norms, stream_norms
from quantized_gradient_compression_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_gradient_compression_b200", "csrc")
EMU = os.path.join(HERE, "emu", "enc")


@pytest.fixture(scope="module")
def enc_exe(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("encemu")
    src_dir = d / "pkg" / "csrc"
    src_dir.mkdir(parents=True)
    shutil.copytree(os.path.join(ROOT, "include"), d / "include")
    for h in ("qsgd_internal.h", "qsgd_limits.h"):
        shutil.copy(os.path.join(CSRC, h), src_dir / h)
    (src_dir / "qsgd_device.cuh").write_text(_host_source(open(os.path.join(CSRC, "qsgd_device.cuh")).read()))
    enc = open(os.path.join(CSRC, "qsgd_encode.cu")).read()
    cut = enc.index("template <int V, bool kShort, bool kEF>\ncudaError_t launch_fast")
    (src_dir / "encode_emu.inc").write_text(_host_source(enc[:cut]) + "}  // namespace\n}  // namespace qsgd\n")
    exe = d / "enc_main"
    r = subprocess.run(["g++", "-O1", "-std=c++17", "-ffp-contract=off", "-pthread", "-I", EMU, "-I", str(src_dir),
                        os.path.join(EMU, "enc_main.cpp"), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    return str(exe)


def _run(exe, tmp, v, d, s, seed, mode, grid, norm_kind=0, e=None):
    n = v.size
    cap = max(1, (32 * ((n + d - 1) // d) + n * (2 + _omega_len(s)) + 31) // 32)
    np.array([n, d, s, seed, norm_kind, 0 if e is None else 1, cap], np.uint64).tofile(tmp / "params.bin")
    v.astype(np.float32).tofile(tmp / "in.bin")
    if e is not None:
        e.astype(np.float32).tofile(tmp / "e_in.bin")
    r = subprocess.run([exe, str(tmp), str(mode), str(grid)], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-500:], r.stderr[-2000:])
    status = int(r.stdout.split()[-1])
    offsets = np.fromfile(tmp / "offsets.bin", np.uint64)
    words = np.fromfile(tmp / "words.bin", np.uint32)[: (int(offsets[-1]) + 31) // 32]
    e_out = np.fromfile(tmp / "e_out.bin", np.float32) if e is not None else None
    return words, offsets, status, e_out


def _omega_len(N):
    length = 1
    while N > 1:
        b = N.bit_length()
        length += b
        N = b - 1
    return length


# (n, d, s, mode, grid, kind): mode 0 encode_fast (d = 128 V; s <= 31 short records,
# s = 64 long), mode 1 encode_general (any d); ragged last buckets and last tiles
CASES = [
    (40_003, 512, 16, 0, 3, "layered"),
    (20_000, 128, 4, 0, 2, "normal"),
    (30_001, 1024, 64, 0, 2, "normal"),
    (9_000, 256, 1, 0, 3, "heavy_tailed_sparse"),
    (7_000, 300, 7, 1, 2, "normal"),
    (20_011, 100, 16, 1, 3, "layered"),
    (12_000, 6000, 2, 1, 2, "normal"),
]


@pytest.mark.parametrize("n,d,s,mode,grid,kind", CASES, ids=["n%d-d%d-s%d-m%d-g%d-%s" % c for c in CASES])
def test_encoder_matches_oracle(enc_exe, tmp_path, oracle_lib, n, d, s, mode, grid, kind):
    v = W.GENERATORS[kind](n, n % 97)
    words, offsets, status, _ = _run(enc_exe, tmp_path, v, d, s, 5, mode, grid)
    own_words, own_offsets, own_norms, own_status = oracle_lib.encode(v, d, s, 5)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, 5, norms_in=gn)
    assert np.array_equal(offsets, r_offsets)
    assert np.array_equal(words, r_words)


@pytest.mark.parametrize("d,s", [(512, 16), (128, 3)])
def test_encoder_max_norm_matches_oracle(enc_exe, tmp_path, oracle_lib, d, s):
    v = W.layered(20_000, 4)
    words, offsets, status, _ = _run(enc_exe, tmp_path, v, d, s, 8, 0, 2, norm_kind=1)
    r_words, r_offsets, _, rst = oracle_lib.encode(v, d, s, 8, norms_in=oracle_lib.maxnorms(v, d))
    assert status == rst and np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)


@pytest.mark.parametrize("d,s", [(512, 16), (256, 40)])
def test_fused_error_feedback_matches_oracle(enc_exe, tmp_path, oracle_lib, d, s):
    g = W.layered(30_001, 6)
    e = W.normal(30_001, 7) * np.float32(0.05)
    words, offsets, status, e_out = _run(enc_exe, tmp_path, g, d, s, 3, 0, 3, e=e)
    own = oracle_lib.encode_ef(g, e, d, s, 3)
    gn = stream_norms(words, offsets)
    check_norms(gn, own[2])
    r_words, r_offsets, _, _, r_e = oracle_lib.encode_ef(g, e, d, s, 3, norms_in=gn)
    assert status == own[3]
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)
    assert np.array_equal(e_out.view(np.uint32), r_e.view(np.uint32))


def test_special_values(enc_exe, tmp_path, oracle_lib):
    v = W.normal(8_192, 2)
    v[:512] = 0.0
    v[700] = np.inf
    v[1300] = np.nan
    v[1600:2048] = 1e-30
    v[2048:2560] = 3e38
    for mode, d in ((0, 512), (1, 500)):
        words, offsets, status, _ = _run(enc_exe, tmp_path, v, d, 16, 1, mode, 2)
        own_words, own_offsets, own_norms, own_status = oracle_lib.encode(v, d, 16, 1)
        assert status == own_status
        gn = stream_norms(words, offsets)
        check_norms(gn, own_norms)
        r_words, r_offsets, _, _ = oracle_lib.encode(v, d, 16, 1, norms_in=gn)
        assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)

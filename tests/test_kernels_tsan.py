"""The kernels' source under ThreadSanitizer on the CPU emulators (no GPU).

Every CUDA thread is a host thread, and the emulators' barriers, warp primitives and
global atomics are host synchronisation that the sanitizer understands.  So a shared-
or global-memory access that no barrier, warp primitive or atomic orders against
another thread's write is reported as a data race.  (A barrier removed from a copy of
decode_multi is reported as six races.)  The decoders (decode_multi, decode_warp,
the row decoders and the large-bucket decoder) and the encoders (encode_fast across
CTAs, encode_general, and the two-launch encoder's coders and compaction, whose
look-back crosses CTAs) must report none."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from emu_source import host_source
from quantized_gradient_compression_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_gradient_compression_b200", "csrc")
TSAN = ["-O1", "-g", "-fsanitize=thread", "-std=c++17", "-ffp-contract=off", "-pthread"]
ENV = dict(os.environ, TSAN_OPTIONS="halt_on_error=0 report_signal_unsafe=0 history_size=2")


def _have_tsan(tmp):
    if shutil.which("g++") is None:
        return False
    src = tmp / "t.cpp"
    src.write_text("int main() { return 0; }\n")
    ok = subprocess.run(["g++", "-fsanitize=thread", str(src), "-o", str(tmp / "t")], capture_output=True)
    return ok.returncode == 0 and subprocess.run([str(tmp / "t")], capture_output=True).returncode == 0


def _races(r):
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stderr.count("WARNING: ThreadSanitizer: data race"), r.stderr[-3000:]


@pytest.fixture(scope="module")
def dec_tsan(tmp_path_factory):
    d = tmp_path_factory.mktemp("dectsan")
    if not _have_tsan(d):
        pytest.skip("no ThreadSanitizer")
    import test_decoder_emulated as T

    (d / "decode_emu.inc").write_text(T._kernel_source())
    exe = d / "emu"
    r = subprocess.run(["g++", *TSAN, "-I", os.path.join(HERE, "emu", "inc"), "-I", str(d),
                        os.path.join(HERE, "emu", "emu_main.cpp"), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    return str(exe)


@pytest.mark.parametrize("d,s,K,P,acc", [(512, 16, 1, -2, 0), (512, 16, 2, -2, 1), (512, 16, 3, -1, 1),
                                         (100, 7, 2, -2, 1)])
def test_decoders_have_no_race(dec_tsan, tmp_path, oracle_lib, d, s, K, P, acc):
    n = 3000
    for j in range(K):
        w, off, _, _ = oracle_lib.encode(W.normal(n, j), d, s, seed=j)
        np.concatenate([w, np.zeros(1, np.uint32)]).tofile(tmp_path / ("w%d.bin" % j))
        off.tofile(tmp_path / ("o%d.bin" % j))
    np.zeros(n, np.float32).tofile(tmp_path / "out_in.bin")
    np.array([n, d, s, K], np.uint64).tofile(tmp_path / "params.bin")
    r = subprocess.run([dec_tsan, str(tmp_path), str(P), str(acc), "1", "0"], capture_output=True, text=True,
                       timeout=900, env=ENV)
    count, tail = _races(r)
    assert count == 0, tail


@pytest.fixture(scope="module")
def enc_tsan(tmp_path_factory):
    d = tmp_path_factory.mktemp("enctsan")
    if not _have_tsan(d):
        pytest.skip("no ThreadSanitizer")
    src_dir = d / "pkg" / "csrc"
    src_dir.mkdir(parents=True)
    shutil.copytree(os.path.join(ROOT, "include"), d / "include")
    for h in ("qsgd_internal.h", "qsgd_limits.h"):
        shutil.copy(os.path.join(CSRC, h), src_dir / h)
    (src_dir / "qsgd_device.cuh").write_text(host_source(open(os.path.join(CSRC, "qsgd_device.cuh")).read()))
    enc = open(os.path.join(CSRC, "qsgd_encode.cu")).read()
    cut = enc.index("template <int V, bool kShort, bool kEF>\ncudaError_t launch_fast")
    (src_dir / "encode_emu.inc").write_text(host_source(enc[:cut]) + "}  // namespace\n}  // namespace qsgd\n")
    exe = d / "enc"
    emu = os.path.join(HERE, "emu", "enc")
    r = subprocess.run(["g++", *TSAN, "-I", emu, "-I", str(src_dir), os.path.join(emu, "enc_main.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    return str(exe)


@pytest.mark.parametrize("n,d,s,mode,grid", [(20_000, 512, 16, 0, 2), (6_000, 128, 40, 0, 3), (8_000, 100, 7, 1, 2)])
def test_encoders_have_no_race(enc_tsan, tmp_path, n, d, s, mode, grid):
    import test_encoder_emulated as E

    cap = max(1, (32 * ((n + d - 1) // d) + n * (2 + E._omega_len(s)) + 31) // 32)
    np.array([n, d, s, 3, 0, 0, cap], np.uint64).tofile(tmp_path / "params.bin")
    W.normal(n, 1).tofile(tmp_path / "in.bin")
    r = subprocess.run([enc_tsan, str(tmp_path), str(mode), str(grid)], capture_output=True, text=True, timeout=1500,
                       env=ENV)
    count, tail = _races(r)
    assert count == 0, tail


# --- the row decoders and the two-launch encoder ---------------------------------------
@pytest.fixture(scope="module")
def rows_tsan(tmp_path_factory):
    d = tmp_path_factory.mktemp("rowstsan")
    if not _have_tsan(d):
        pytest.skip("no ThreadSanitizer")
    import test_rows_emulated as R

    return R.build_rows_exe(d / "b", TSAN)


@pytest.mark.parametrize("n,d,s,K,acc", [(3_000, 512, 16, 1, 0), (3_000, 512, 300, 1, 1), (3_000, 512, 4, 3, 1),
                                         (5_000, 2048, 4, 2, 1)])
def test_row_decoders_have_no_race(rows_tsan, tmp_path, oracle_lib, n, d, s, K, acc):
    """decode_rows, decode_rows_ring, decode_rows_multi and decode_sparse."""
    for j in range(K):
        w, off, _, _ = oracle_lib.encode(W.normal(n, j), d, s, seed=j)
        np.concatenate([w, np.zeros(1, np.uint32)]).tofile(tmp_path / ("w%d.bin" % j))
        off.tofile(tmp_path / ("o%d.bin" % j))
    np.zeros(n, np.float32).tofile(tmp_path / "out_in.bin")
    np.array([n, d, s], np.uint64).tofile(tmp_path / "params.bin")
    r = subprocess.run([rows_tsan, str(tmp_path), str(acc), "2", "2", str(K), "0"], capture_output=True, text=True,
                       timeout=900, env=ENV)
    count, tail = _races(r)
    assert count == 0, tail


@pytest.fixture(scope="module")
def stage_tsan(tmp_path_factory):
    d = tmp_path_factory.mktemp("stagetsan")
    if not _have_tsan(d):
        pytest.skip("no ThreadSanitizer")
    import test_stage_emulated as S

    # compaction tiles of 32 buckets: the look-back crosses CTAs several times
    return S._build(tmp_path_factory, "stagetsanb", [*TSAN, "-DQSGD_COMPACT_BLOCK=32"])


@pytest.mark.parametrize("n,d,s,grid", [(20_000, 512, 16, 2), (6_000, 128, 40, 3), (12_000, 4096, 2, 2)])
def test_staged_encoder_has_no_race(stage_tsan, tmp_path, n, d, s, grid):
    import test_stage_emulated as S

    cap = max(1, (32 * ((n + d - 1) // d) + n * (2 + S._omega_len(s)) + 31) // 32)
    np.array([n, d, s, 3, 0, 0, cap], np.uint64).tofile(tmp_path / "params.bin")
    W.normal(n, 1).astype(np.float32).tofile(tmp_path / "in.bin")
    r = subprocess.run([stage_tsan, str(tmp_path), str(grid)], capture_output=True, text=True, timeout=1500, env=ENV)
    count, tail = _races(r)
    assert count == 0, tail

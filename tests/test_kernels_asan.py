"""The kernels' source under AddressSanitizer on the CPU emulators (no GPU).

- Decoders on damaged input: random bit flips anywhere (norm fields included),
  scrambled offsets headers, and word arrays cut short -- decode_multi and
  decode_warp, and the row decoders (decode_rows, decode_rows_ring,
  decode_rows_multi) with the large-bucket decoder (decode_sparse).  They may flag
  the input, but they must read and write nothing outside their buffers, and must
  end.
- Encoders at ragged shapes and special values -- the one-pass encode_fast and
  encode_general, and the two-launch encoder (code_buckets_short, code_buckets,
  compact_stream): every access stays in bounds, and the stream still matches the
  oracle."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from emu_source import host_source
from gpu_common import check_norms, stream_norms
from quantized_gradient_compression_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_gradient_compression_b200", "csrc")
ASAN = ["-O1", "-g", "-fsanitize=address", "-fno-omit-frame-pointer", "-std=c++17", "-ffp-contract=off", "-pthread"]


def _have_asan(tmp):
    if shutil.which("g++") is None:
        return False
    src = tmp / "t.cpp"
    src.write_text("int main() { return 0; }\n")
    return subprocess.run(["g++", "-fsanitize=address", str(src), "-o", str(tmp / "t")],
                          capture_output=True).returncode == 0


@pytest.fixture(scope="module")
def dec_asan(tmp_path_factory):
    d = tmp_path_factory.mktemp("decasan")
    if not _have_asan(d):
        pytest.skip("no AddressSanitizer")
    import test_decoder_emulated as T

    (d / "decode_emu.inc").write_text(T._kernel_source())
    exe = d / "emu"
    r = subprocess.run(["g++", *ASAN, "-I", os.path.join(HERE, "emu", "inc"), "-I", str(d),
                        os.path.join(HERE, "emu", "emu_main.cpp"), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    return str(exe)


def test_decoders_on_damaged_input(dec_asan, tmp_path, oracle_lib):
    rng = np.random.default_rng(2024)
    for trial in range(40):
        n = int(rng.integers(1, 6000))
        d = int(rng.choice([4, 64, 100, 128, 512, 1000, 4096]))
        s = int(rng.choice([1, 3, 16, 100, 1023]))
        K = int(rng.integers(1, 4))
        P = int(rng.choice([-1, -2]))
        acc = bool(rng.integers(0, 2)) or P == -1
        t = tmp_path / ("t%d" % trial)
        t.mkdir()
        for j in range(K):
            words, offsets, _, _ = oracle_lib.encode(W.normal(n, trial * 10 + j), d, s, seed=j)
            mode = rng.integers(0, 4)
            if mode == 0 and words.size:
                for pos in rng.integers(0, words.size * 32, size=8):
                    words[pos >> 5] ^= np.uint32(1) << np.uint32(31 - (pos & 31))
            elif mode == 1:
                offsets = offsets.copy()
                idx = rng.integers(0, offsets.size, size=3)
                offsets[idx] = rng.integers(0, max(1, int(offsets[-1]) * 2 + 64), size=3).astype(np.uint64)
            elif mode == 2 and words.size > 2:
                words = words[: max(1, words.size // 2)]
            words.astype(np.uint32).tofile(t / ("w%d.bin" % j))
            offsets.astype(np.uint64).tofile(t / ("o%d.bin" % j))
        np.zeros(n, np.float32).tofile(t / "out_in.bin")
        np.array([n, d, s, K], np.uint64).tofile(t / "params.bin")
        r = subprocess.run([dec_asan, str(t), str(P), "1" if acc else "0", "2", "0"], capture_output=True,
                           text=True, timeout=600)
        assert r.returncode == 0 and "AddressSanitizer" not in r.stderr, (trial, n, d, s, K, P, r.stderr[-2000:])


@pytest.fixture(scope="module")
def enc_asan(tmp_path_factory):
    d = tmp_path_factory.mktemp("encasan")
    if not _have_asan(d):
        pytest.skip("no AddressSanitizer")
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
    r = subprocess.run(["g++", *ASAN, "-I", emu, "-I", str(src_dir), os.path.join(emu, "enc_main.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    return str(exe)


@pytest.mark.parametrize("n,d,s,mode,special", [(5_003, 512, 16, 0, True), (3_001, 128, 40, 0, False),
                                                (4_097, 1024, 3, 0, False), (2_501, 77, 9, 1, True),
                                                (1, 512, 16, 0, False), (9, 5000, 2, 1, False)])
def test_encoders_stay_in_bounds(enc_asan, tmp_path, oracle_lib, n, d, s, mode, special):
    import test_encoder_emulated as E

    v = W.normal(n, 4)
    if special and n > 1800:
        v[:300] = 0.0
        v[400] = np.inf
        v[900] = np.nan
        v[1200:1500] = 1e-30
        v[1500:1800] = 3e38
    words, offsets, status, _ = E._run(enc_asan, tmp_path, v, d, s, 2, mode, 2)
    own_words, own_offsets, own_norms, own_status = oracle_lib.encode(v, d, s, 2)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, 2, norms_in=gn)
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)


# --- the row decoders, the several-stream tiles and the large-bucket decoder --------
@pytest.fixture(scope="module")
def rows_asan(tmp_path_factory):
    d = tmp_path_factory.mktemp("rowsasan")
    if not _have_asan(d):
        pytest.skip("no AddressSanitizer")
    import test_rows_emulated as R

    return R.build_rows_exe(d / "b", ASAN)


def test_row_decoders_on_damaged_input(rows_asan, tmp_path, oracle_lib):
    """decode_rows (byte codes), decode_rows_ring (16-bit codes), decode_rows_multi
    and decode_rows_side (K > 1), and decode_sparse (d > 1024) on bit flips, scrambled
    offsets and cut word arrays: they may flag the input, but touch nothing outside
    their buffers."""
    rng = np.random.default_rng(77)
    for trial in range(40):
        n = int(rng.integers(1, 6000))
        d = int(rng.choice([4, 100, 512, 1000, 1024, 2048, 3001]))
        s = int(rng.choice([1, 3, 16, 127, 300, 32767]))
        K = int(rng.integers(1, 4)) if d <= 1024 else int(rng.integers(1, 3))
        acc = bool(rng.integers(0, 2))
        t = tmp_path / ("t%d" % trial)
        t.mkdir()
        for j in range(K):
            words, offsets, _, _ = oracle_lib.encode(W.normal(n, trial * 10 + j), d, s, seed=j)
            mode = rng.integers(0, 4)
            if mode == 0 and words.size:
                for pos in rng.integers(0, words.size * 32, size=8):
                    words[pos >> 5] ^= np.uint32(1) << np.uint32(31 - (pos & 31))
            elif mode == 1:
                offsets = offsets.copy()
                idx = rng.integers(0, offsets.size, size=3)
                offsets[idx] = rng.integers(0, max(1, int(offsets[-1]) * 2 + 64), size=3).astype(np.uint64)
            elif mode == 2 and words.size > 2:
                words = words[: max(1, words.size // 2)]
            words.astype(np.uint32).tofile(t / ("w%d.bin" % j))
            offsets.astype(np.uint64).tofile(t / ("o%d.bin" % j))
        np.zeros(n, np.float32).tofile(t / "out_in.bin")
        np.array([n, d, s], np.uint64).tofile(t / "params.bin")
        side = d <= 1024 and s <= 127 and K > 1 and trial % 2 == 1
        r = subprocess.run([rows_asan, str(t), "1" if acc else "0", "2", "2", str(K), "0", "1" if side else "0"],
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0 and "AddressSanitizer" not in r.stderr, (trial, n, d, s, K, r.stderr[-2000:])


# --- the two-launch encoder (bucket coders and compaction) ----------------------------
@pytest.fixture(scope="module")
def stage_asan(tmp_path_factory):
    d = tmp_path_factory.mktemp("stageasan")
    if not _have_asan(d):
        pytest.skip("no AddressSanitizer")
    import test_stage_emulated as S

    return S._build(tmp_path_factory, "stageasanb", ASAN)


@pytest.mark.parametrize("n,d,s,special", [(5_003, 512, 16, True), (3_001, 128, 40, False), (9_001, 4096, 2, True),
                                           (2_501, 4, 9, False), (1, 512, 16, False), (20_000, 1000, 31, False)])
def test_staged_encoder_stays_in_bounds(stage_asan, tmp_path, oracle_lib, n, d, s, special):
    import test_stage_emulated as S

    v = W.normal(n, 5)
    if special and n > 1800:
        v[:300] = 0.0
        v[400] = np.inf
        v[900] = np.nan
        v[1200:1500] = 1e-30
        v[1500:1800] = 3e38
    words, offsets, status, _ = S._run(stage_asan, tmp_path, v, d, s, 2, 2)
    _, _, own_norms, own_status = oracle_lib.encode(v, d, s, 2)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, 2, norms_in=gn)
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)

"""The two-launch encoder's exact source (code_buckets, then compact_stream) on the
CPU block emulator (no GPU).

Each grid runs with all its CTAs at once, every CUDA thread a host thread; warp
primitives check that their 32 lanes meet at the same call site.  The workspace is
filled with garbage past the control block first, so the kernels may rely only on
what they write themselves.  The stream and offsets are compared bit for bit with the
oracle's encode under the emulated encoder's own norms (the wire format lets an
encoder choose its fp32 norm within 1e-6); the memory with the oracle's
error-feedback encode."""

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


def _build(tmp_path_factory, name, extra=()):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp(name)
    src_dir = d / "pkg" / "csrc"
    src_dir.mkdir(parents=True)
    shutil.copytree(os.path.join(ROOT, "include"), d / "include")
    for h in ("qsgd_internal.h", "qsgd_limits.h"):
        shutil.copy(os.path.join(CSRC, h), src_dir / h)
    (src_dir / "qsgd_device.cuh").write_text(_host_source(open(os.path.join(CSRC, "qsgd_device.cuh")).read()))
    enc = open(os.path.join(CSRC, "qsgd_encode_stage.cu")).read()
    cut = enc.index("// One instance per kernel, so that each kernel gets its own shared-memory attribute.")
    (src_dir / "stage_emu.inc").write_text(_host_source(enc[:cut]) + "}  // namespace\n}  // namespace qsgd\n")
    exe = d / "stage_main"
    r = subprocess.run(["g++", "-O1", "-std=c++17", "-ffp-contract=off", "-pthread", *extra, "-I", EMU, "-I",
                        str(src_dir), os.path.join(EMU, "stage_main.cpp"), "-o", str(exe)], capture_output=True,
                       text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    return str(exe)


@pytest.fixture(scope="module")
def stage_exe(tmp_path_factory):
    return _build(tmp_path_factory, "stageemu")


@pytest.fixture(scope="module")
def stage_exe_direct(tmp_path_factory):
    # a shared-memory gather of 64 words: nearly every tile reads the staging slots
    # directly, the path of tiles too large to gather
    return _build(tmp_path_factory, "stageemudirect", ["-DQSGD_COMPACT_SMEM_WORDS=64"])


@pytest.fixture(scope="module")
def stage_exe_small_tiles(tmp_path_factory):
    # compaction tiles of 32 buckets, so that the look-back walks several windows
    return _build(tmp_path_factory, "stageemu32", ["-DQSGD_COMPACT_BLOCK=32"])


def _omega_len(N):
    length = 1
    while N > 1:
        b = N.bit_length()
        length += b
        N = b - 1
    return length


def _run(exe, tmp, v, d, s, seed, grid, norm_kind=0, e=None):
    n = v.size
    cap = max(1, (32 * ((n + d - 1) // d) + n * (2 + _omega_len(s)) + 31) // 32)
    np.array([n, d, s, seed, norm_kind, 0 if e is None else 1, cap], np.uint64).tofile(tmp / "params.bin")
    v.astype(np.float32).tofile(tmp / "in.bin")
    if e is not None:
        e.astype(np.float32).tofile(tmp / "e_in.bin")
    r = subprocess.run([exe, str(tmp), str(grid)], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-500:], r.stderr[-2000:])
    status = int(r.stdout.split()[-1])
    offsets = np.fromfile(tmp / "offsets.bin", np.uint64)
    words = np.fromfile(tmp / "words.bin", np.uint32)[: (int(offsets[-1]) + 31) // 32]
    e_out = np.fromfile(tmp / "e_out.bin", np.float32) if e is not None else None
    return words, offsets, status, e_out


# (n, d, s, grid, kind): every lane count per bucket (d = 4 .. 1024), both record
# kinds (s <= 31 whole-record table, larger s omega table), ragged last buckets and
# more than one compaction tile (nb > 256)
CASES = [
    (40_003, 512, 16, 3, "layered"),
    (20_000, 128, 4, 2, "normal"),
    (30_001, 1024, 64, 2, "normal"),
    (9_000, 256, 1, 3, "heavy_tailed_sparse"),
    (70_001, 200, 7, 2, "normal"),
    (3_001, 4, 2, 1, "normal"),
    (5_000, 384, 3000, 1, "normal"),
    # levels whose codes make a lane's run longer than 96 bits, and codes past 31 bits
    (4_000, 128, 1 << 20, 1, "normal"),
    (4_000, 256, 1 << 22, 1, "normal"),
    (6_000, 1000, 31, 2, "layered"),
    (1, 512, 16, 1, "normal"),
    # buckets of several 512-coordinate chunks (s <= 31): whole, ragged and partial chunks
    (60_001, 8192, 1, 2, "heavy_tailed_sparse"),
    (40_003, 3000, 16, 2, "layered"),
    (50_000, 16384, 4, 2, "normal"),
]


@pytest.mark.parametrize("n,d,s,grid,kind", CASES, ids=["n%d-d%d-s%d-g%d-%s" % c for c in CASES])
def test_stage_encoder_matches_oracle(stage_exe, tmp_path, oracle_lib, n, d, s, grid, kind):
    v = W.GENERATORS[kind](n, n % 97)
    words, offsets, status, _ = _run(stage_exe, tmp_path, v, d, s, 5, grid)
    _, _, own_norms, own_status = oracle_lib.encode(v, d, s, 5)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, 5, norms_in=gn)
    assert np.array_equal(offsets, r_offsets)
    assert np.array_equal(words, r_words)


@pytest.mark.parametrize("n,d,s,grid,kind", CASES[:6], ids=["n%d-d%d-s%d-g%d-%s" % c for c in CASES[:6]])
def test_stage_encoder_direct_copy_matches_oracle(stage_exe_direct, tmp_path, oracle_lib, n, d, s, grid, kind):
    """The compaction's copy from the staging slots (tiles too large for its
    shared-memory gather)."""
    v = W.GENERATORS[kind](n, n % 97)
    words, offsets, status, _ = _run(stage_exe_direct, tmp_path, v, d, s, 5, grid)
    _, _, own_norms, own_status = oracle_lib.encode(v, d, s, 5)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, 5, norms_in=gn)
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)


@pytest.mark.parametrize("d,s", [(512, 16), (128, 3), (256, 100), (4096, 8)])
def test_stage_encoder_max_norm_matches_oracle(stage_exe, tmp_path, oracle_lib, d, s):
    v = W.layered(20_000, 4)
    words, offsets, status, _ = _run(stage_exe, tmp_path, v, d, s, 8, 2, norm_kind=1)
    r_words, r_offsets, _, rst = oracle_lib.encode(v, d, s, 8, norms_in=oracle_lib.maxnorms(v, d))
    assert status == rst and np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)


@pytest.mark.parametrize("d,s", [(512, 16), (256, 40), (100, 5), (2048, 3)])
def test_stage_error_feedback_matches_oracle(stage_exe, tmp_path, oracle_lib, d, s):
    g = W.layered(30_001, 6)
    e = W.normal(30_001, 7) * np.float32(0.05)
    e[:d] = np.nan  # a non-finite bucket: sent as zero, its memory keeps p
    words, offsets, status, e_out = _run(stage_exe, tmp_path, g, d, s, 3, 3, e=e)
    own = oracle_lib.encode_ef(g, e, d, s, 3)
    gn = stream_norms(words, offsets)
    check_norms(gn, own[2])
    r_words, r_offsets, _, _, r_e = oracle_lib.encode_ef(g, e, d, s, 3, norms_in=gn)
    assert status == own[3]
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)
    assert np.array_equal(e_out.view(np.uint32), r_e.view(np.uint32))


def test_stage_special_values(stage_exe, tmp_path, oracle_lib):
    v = W.normal(8_192, 2)
    v[:512] = 0.0
    v[700] = np.inf
    v[1300] = np.nan
    v[1600:2048] = 1e-30
    v[2048:2560] = 3e38
    v[3000:3512] = -0.0
    for d in (512, 500, 4096):
        words, offsets, status, _ = _run(stage_exe, tmp_path, v, d, 16, 1, 2)
        _, _, own_norms, own_status = oracle_lib.encode(v, d, 16, 1)
        assert status == own_status
        gn = stream_norms(words, offsets)
        check_norms(gn, own_norms)
        r_words, r_offsets, _, _ = oracle_lib.encode(v, d, 16, 1, norms_in=gn)
        assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)


def test_stage_lane_strings_past_96_bits(stage_exe, tmp_path, oracle_lib):
    """A lane whose 16 coordinates all carry large levels needs more than 96 bits for
    its records (the short coder's register string): the bucket is then placed record
    by record, and the stream must not change."""
    v = (W.normal(8_192, 3) * np.float32(1e-3)).astype(np.float32)
    for b in range(0, 8_192, 512):
        lane = (b // 512) % 32
        v[b + 16 * lane: b + 16 * lane + 16] = np.float32(1.0)  # norm ~4: levels ~8 at s = 31
    words, offsets, status, _ = _run(stage_exe, tmp_path, v, 512, 31, 2, 2)
    _, _, own_norms, own_status = oracle_lib.encode(v, 512, 31, 2)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, 512, 31, 2, norms_in=gn)
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)
    assert int(np.diff(offsets.astype(np.int64)).max()) > 32 + 96  # some bucket took the record-by-record path


@pytest.mark.parametrize("n,d,s", [(12_000, 4, 3), (40_003, 128, 16)])
def test_stage_lookback_over_several_windows(stage_exe_small_tiles, tmp_path, oracle_lib, n, d, s):
    """Compaction tiles of 32 buckets (CTAs of 64 threads): 94 and 10 tiles, so a
    tile's look-back reads up to two windows of 64 predecessors before it meets a
    prefix."""
    v = W.layered(n, 5)
    words, offsets, status, _ = _run(stage_exe_small_tiles, tmp_path, v, d, s, 4, 2)
    _, _, own_norms, own_status = oracle_lib.encode(v, d, s, 4)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, 4, norms_in=gn)
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)


def test_stage_compaction_tiles_on_both_paths(stage_exe, tmp_path, oracle_lib):
    """Tiles of 256 buckets at s = 48: full tiles hold about 16,920 staged words,
    more than the compaction's shared-memory gather, so they copy from the staging
    slots; tiles with zero buckets hold fewer and are gathered."""
    n = 3 * 256 * 512
    v = W.normal(n, 3)
    v[256 * 512:256 * 512 + 60 * 512] = 0.0
    words, offsets, status, _ = _run(stage_exe, tmp_path, v, 512, 48, 1, 3)
    _, _, own_norms, own_status = oracle_lib.encode(v, 512, 48, 1)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, 512, 48, 1, norms_in=gn)
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)


def test_stage_compaction_with_unaligned_slots(stage_exe, tmp_path, oracle_lib, monkeypatch):
    """Staging slots laid out word by word (not the library's layout): the compaction
    must not gather them 16 bytes a copy (the emulator rejects an unaligned 16-byte
    copy) and must still place every bit."""
    monkeypatch.setenv("STAGE_UNPADDED", "1")
    n, d, s = 20_003, 100, 7  # 32 + 100 * (2 + 6) bits: 26 words a slot
    v = W.normal(n, 8)
    words, offsets, status, _ = _run(stage_exe, tmp_path, v, d, s, 2, 2)
    _, _, own_norms, own_status = oracle_lib.encode(v, d, s, 2)
    assert status == own_status
    gn = stream_norms(words, offsets)
    check_norms(gn, own_norms)
    r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, 2, norms_in=gn)
    assert np.array_equal(offsets, r_offsets) and np.array_equal(words, r_words)


"""The one-stream row decoder's exact source (decode_rows) on the CPU block emulator
(no GPU).

All CTAs of a launch run at once, every CUDA thread a host thread; warp primitives
check that their 32 lanes meet at the same call site, and shared memory starts as
garbage.  Streams come from the oracle's encoder; the output is compared bit for bit
with the oracle's decode (or decode-accumulate onto an output holding -0.0 values).
Bit flips in some buckets must be flagged, and every bucket no flip touched must
still decode as the oracle decodes it."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from emu_source import host_source as _host_source
from quantized_gradient_compression_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_gradient_compression_b200", "csrc")
EMU = os.path.join(HERE, "emu", "enc")


def build_rows_exe(d, extra=()):
    """Builds the row decoders' host program in directory d (extra: g++ flags)."""
    src_dir = d / "pkg" / "csrc"
    src_dir.mkdir(parents=True)
    shutil.copytree(os.path.join(ROOT, "include"), d / "include")
    for h in ("qsgd_internal.h", "qsgd_limits.h"):
        shutil.copy(os.path.join(CSRC, h), src_dir / h)
    (src_dir / "qsgd_device.cuh").write_text(_host_source(open(os.path.join(CSRC, "qsgd_device.cuh")).read()))
    (src_dir / "qsgd_tables.cuh").write_text(_host_source(open(os.path.join(CSRC, "qsgd_tables.cuh")).read()))
    src = open(os.path.join(CSRC, "qsgd_decode_rows.cu")).read()
    cut = src.index("// One CTA per SM, its warps one group each where the groups allow: every SM busy.")
    (src_dir / "rows_emu.inc").write_text(_host_source(src[:cut]) + "}  // namespace\n}  // namespace qsgd\n")
    exe = d / "rows_main"
    flags = list(extra) or ["-O1"]
    r = subprocess.run(["g++", *flags, "-std=c++17", "-ffp-contract=off", "-pthread", "-I", EMU, "-I", str(src_dir),
                        os.path.join(EMU, "rows_main.cpp"), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    return str(exe)


@pytest.fixture(scope="module")
def rows_exe(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    return build_rows_exe(tmp_path_factory.mktemp("rowsemu"))


def _flip_bits(words, offsets, rng):
    nb = offsets.size - 1
    for b in rng.integers(0, nb, size=max(1, nb // 8)):
        lo, hi = int(offsets[b]) + 32, int(offsets[b + 1])
        if hi > lo:
            for pos in rng.integers(lo, hi, size=3):
                words[pos >> 5] ^= np.uint32(1) << np.uint32(31 - (pos & 31))


def _run(exe, tmp, words, offsets, n, d, s, accumulate, grid, warps, base):
    np.concatenate([words, np.zeros(1, np.uint32)]).tofile(tmp / "w0.bin")
    offsets.astype(np.uint64).tofile(tmp / "o0.bin")
    base.tofile(tmp / "out_in.bin")
    np.array([n, d, s], np.uint64).tofile(tmp / "params.bin")
    r = subprocess.run([exe, str(tmp), "1" if accumulate else "0", str(grid), str(warps)],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, (r.stdout[-500:], r.stderr[-2000:])
    return np.fromfile(tmp / "out.bin", np.float32), int(r.stdout.split()[-1])


def _base(n, d, accumulate):
    base = (np.random.default_rng(d).standard_normal(n) * 1e-3).astype(np.float32)
    base[::5] = np.float32(-0.0)
    if not accumulate:
        base[:] = np.float32(np.nan)  # every coordinate must be written
    return base


# (n, d, s, accumulate, grid, warps, input): every lane count per row (d = 4 .. 1024),
# ragged last bucket and last group, sparse streams with long records (bit-serial
# path), s up to 127, warps that take several groups
CASES = [
    (40_003, 512, 16, False, 2, 3, "layered"),
    (40_003, 512, 16, True, 2, 3, "layered"),
    (20_000, 128, 4, False, 1, 4, "normal"),
    (30_001, 1024, 64, True, 2, 2, "normal"),
    (9_000, 256, 1, False, 2, 2, "heavy_tailed_sparse"),
    (70_001, 200, 7, True, 3, 2, "normal"),
    (3_001, 4, 2, False, 2, 2, "normal"),
    (6_000, 1000, 127, False, 1, 2, "layered"),
    (1, 512, 16, True, 1, 1, "normal"),
    # gaps past the ring of two segments (records held back until their segment)
    (20_000, 1024, 1, False, 2, 2, "heavy_tailed_sparse"),
    (20_000, 1024, 200, True, 2, 2, "heavy_tailed_sparse"),
    # 16-bit codes (s > 127): large levels, and records the table never holds
    (20_000, 512, 256, False, 2, 2, "normal"),
    (20_000, 512, 256, True, 2, 2, "layered"),
    (9_001, 100, 32767, False, 1, 3, "normal"),
]


@pytest.mark.parametrize("n,d,s,accumulate,grid,warps,kind", CASES,
                         ids=["n%d-d%d-s%d-acc%d-g%d-w%d-%s" % c for c in CASES])
def test_row_decoder_matches_oracle(rows_exe, tmp_path, oracle_lib, n, d, s, accumulate, grid, warps, kind):
    v = W.GENERATORS[kind](n, n % 89)
    words, offsets, _, st = oracle_lib.encode(v, d, s, seed=11)
    assert st == 0
    base = _base(n, d, accumulate)
    got, status = _run(rows_exe, tmp_path, words, offsets, n, d, s, accumulate, grid, warps, base)
    assert status == 0
    if accumulate:
        ref = base.copy()
        _, rst = oracle_lib.decode_accumulate([(words, offsets)], n, d, s, ref)
    else:
        ref, rst = oracle_lib.decode(words, offsets, n, d, s)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("d,s", [(1024, 16), (1000, 300)])
def test_row_decoder_far_records(rows_exe, tmp_path, oracle_lib, d, s):
    """Buckets whose first record lies more than two segments ahead (a bit-serial
    gap, held back until its segment), next to dense buckets."""
    n = 64 * d
    rng = np.random.default_rng(d)
    v = np.zeros(n, np.float32)
    for b in range(0, 64, 2):
        pos = rng.integers(300, d, size=2)
        v[b * d + pos] = rng.standard_normal(2).astype(np.float32)
        v[(b + 1) * d:(b + 2) * d] = rng.standard_normal(d).astype(np.float32)
    words, offsets, _, st = oracle_lib.encode(v, d, s, seed=4)
    assert st == 0
    got, status = _run(rows_exe, tmp_path, words, offsets, n, d, s, False, 2, 2, _base(n, d, False))
    ref, rst = oracle_lib.decode(words, offsets, n, d, s)
    assert status == 0 and rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("d,accumulate,s", [(512, False, 16), (128, True, 16), (1000, False, 16), (512, True, 300),
                                          (256, False, 2)])
def test_row_decoder_corrupt_streams(rows_exe, tmp_path, oracle_lib, d, accumulate, s):
    n = 30_000
    v = W.normal(n, 5)
    intact, offsets, _, _ = oracle_lib.encode(v, d, s, seed=3)
    words = intact.copy()
    _flip_bits(words, offsets, np.random.default_rng(d))
    base = _base(n, d, accumulate)
    got, status = _run(rows_exe, tmp_path, words, offsets, n, d, s, accumulate, 2, 2, base)
    assert status & 2
    if accumulate:
        ref = base.copy()
        oracle_lib.decode_accumulate([(intact, offsets)], n, d, s, ref)
    else:
        ref, _ = oracle_lib.decode(intact, offsets, n, d, s)
    flipped = words != intact
    keep = np.ones(n, dtype=bool)
    for b in range(offsets.size - 1):
        w0, w1 = int(offsets[b]) >> 5, (int(offsets[b + 1]) + 31) >> 5
        if flipped[w0:w1].any():
            keep[b * d:min(n, (b + 1) * d)] = False
    assert keep.any() and not keep.all()
    assert np.array_equal(got[keep].view(np.uint32), ref[keep].view(np.uint32))


# decode_rows_multi: K streams added onto fp32 tiles in stream order, decode-accumulate
# and the mean; past one launch (16 streams); sparse and dense streams, ragged shapes
MULTI = [
    (20_003, 512, 4, 3, False, "small_normal"),
    (20_003, 512, 16, 2, True, "layered"),
    (9_001, 128, 4, 17, False, "small_normal"),
    (7_000, 100, 7, 5, True, "normal"),
    (5_000, 1000, 300, 3, False, "normal"),
    (3_000, 512, 1, 18, True, "heavy_tailed_sparse"),
]


def _run_multi(exe, tmp, streams, n, d, s, mean, base, grid=2, warps=2, side=False):
    for j, (w, o) in enumerate(streams):
        np.concatenate([w, np.zeros(1, np.uint32)]).tofile(tmp / ("w%d.bin" % j))
        o.astype(np.uint64).tofile(tmp / ("o%d.bin" % j))
    base.tofile(tmp / "out_in.bin")
    np.array([n, d, s], np.uint64).tofile(tmp / "params.bin")
    r = subprocess.run([exe, str(tmp), "1", str(grid), str(warps), str(len(streams)), "1" if mean else "0",
                        "1" if side else "0"], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-500:], r.stderr[-2000:])
    return np.fromfile(tmp / "out.bin", np.float32), int(r.stdout.split()[-1])


@pytest.mark.parametrize("n,d,s,K,mean,kind", MULTI, ids=["n%d-d%d-s%d-K%d-mean%d-%s" % c for c in MULTI])
def test_row_multi_decoder_matches_oracle(rows_exe, tmp_path, oracle_lib, n, d, s, K, mean, kind):
    streams = []
    for j in range(K):
        v = W.GENERATORS[kind](n, 50 + j)
        w, o, _, st = oracle_lib.encode(v, d, s, seed=j)
        assert st == 0
        streams.append((w, o))
    base = _base(n, d, True)
    got, status = _run_multi(rows_exe, tmp_path, streams, n, d, s, mean, base)
    assert status == 0
    if mean:
        ref, rst = oracle_lib.decode_mean(streams, n, d, s)
    else:
        ref = base.copy()
        _, rst = oracle_lib.decode_accumulate(streams, n, d, s, ref)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_row_multi_decoder_corrupt_stream(rows_exe, tmp_path, oracle_lib):
    n, d, s, K = 20_000, 512, 4, 3
    intact, streams = [], []
    for j in range(K):
        w, o, _, _ = oracle_lib.encode(W.small_normal(n, 70 + j), d, s, seed=j)
        intact.append((w, o))
        w2 = w.copy()
        if j == 1:
            _flip_bits(w2, o, np.random.default_rng(9))
        streams.append((w2, o))
    base = _base(n, d, True)
    got, status = _run_multi(rows_exe, tmp_path, streams, n, d, s, False, base)
    assert status & 2
    ref = base.copy()
    oracle_lib.decode_accumulate(intact, n, d, s, ref)
    keep = np.ones(n, dtype=bool)
    flipped = streams[1][0] != intact[1][0]
    offs = intact[1][1]
    for b in range(offs.size - 1):
        w0, w1 = int(offs[b]) >> 5, (int(offs[b + 1]) + 31) >> 5
        if flipped[w0:w1].any():
            keep[b * d:min(n, (b + 1) * d)] = False
    assert keep.any() and not keep.all()
    assert np.array_equal(got[keep].view(np.uint32), ref[keep].view(np.uint32))


# decode_rows_side: K streams parsed side by side (a warp a stream) into rings of byte
# codes, added onto the output in stream order after each segment.  K from one (the
# mean) past a chunk of eight warps and past one launch of 16; every d % 128 class and
# a ragged last bucket; grids that leave CTAs several sets of groups (the rings are
# reused); sparse streams with gaps past the ring (bit-serial records held back).
SIDE = [
    (20_003, 512, 4, 2, False, 1, "small_normal"),
    (20_003, 512, 16, 3, True, 2, "layered"),
    (9_001, 128, 4, 17, False, 2, "small_normal"),
    (7_000, 100, 7, 5, True, 1, "normal"),
    (6_000, 1000, 127, 8, False, 2, "layered"),
    (6_000, 1024, 16, 9, True, 1, "normal"),
    (3_000, 512, 1, 18, True, 2, "heavy_tailed_sparse"),
    (4_000, 4, 2, 4, False, 1, "normal"),
    (12_000, 200, 16, 1, True, 1, "layered"),
    (30_000, 1024, 1, 2, False, 1, "heavy_tailed_sparse"),
    (1, 512, 16, 2, False, 1, "normal"),
]


@pytest.mark.parametrize("n,d,s,K,mean,grid,kind", SIDE, ids=["n%d-d%d-s%d-K%d-mean%d-g%d-%s" % c for c in SIDE])
def test_side_decoder_matches_oracle(rows_exe, tmp_path, oracle_lib, n, d, s, K, mean, grid, kind):
    streams = []
    for j in range(K):
        v = W.GENERATORS[kind](n, 90 + j)
        w, o, _, st = oracle_lib.encode(v, d, s, seed=3 + j)
        assert st == 0
        streams.append((w, o))
    base = _base(n, d, True)
    got, status = _run_multi(rows_exe, tmp_path, streams, n, d, s, mean, base, grid=grid, side=True)
    assert status == 0
    if mean:
        ref, rst = oracle_lib.decode_mean(streams, n, d, s)
    else:
        ref = base.copy()
        _, rst = oracle_lib.decode_accumulate(streams, n, d, s, ref)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.fixture(scope="module")
def rows_exe_seg128(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    return build_rows_exe(tmp_path_factory.mktemp("rowsemu128"), ("-O1", "-DQSGD_SIDE_SEG=128"))


@pytest.mark.parametrize("n,d,s,K,mean,grid,kind", [SIDE[1], SIDE[6], SIDE[9]],
                         ids=["n%d-d%d-s%d-K%d-mean%d-g%d-%s" % c for c in (SIDE[1], SIDE[6], SIDE[9])])
def test_side_decoder_128_column_segments(rows_exe_seg128, tmp_path, oracle_lib, n, d, s, K, mean, grid, kind):
    """The same kernel built with segments of 128 columns (two CTAs an SM)."""
    test_side_decoder_matches_oracle(rows_exe_seg128, tmp_path, oracle_lib, n, d, s, K, mean, grid, kind)


@pytest.fixture(scope="module")
def rows_exe_ring64(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    return build_rows_exe(tmp_path_factory.mktemp("rowsemuring64"), ("-O1", "-DQSGD_ROWS_SEG=64"))


RING = [c for c in CASES if c[2] > 127]


@pytest.mark.parametrize("n,d,s,accumulate,grid,warps,kind", RING, ids=["n%d-d%d-s%d-acc%d-g%d-w%d-%s" % c for c in RING])
def test_ring_decoder_64_column_segments(rows_exe_ring64, tmp_path, oracle_lib, n, d, s, accumulate, grid, warps, kind):
    """The 16-bit ring decoder built with segments of 64 columns (two rows a pass)."""
    test_row_decoder_matches_oracle(rows_exe_ring64, tmp_path, oracle_lib, n, d, s, accumulate, grid, warps, kind)


def test_side_decoder_far_records(rows_exe, tmp_path, oracle_lib):
    """Buckets whose records lie more than two segments ahead (bit-serial gaps held
    back until their segment), next to dense buckets, in three streams."""
    d, s = 1024, 16
    n = 64 * d
    streams = []
    for j in range(3):
        rng = np.random.default_rng(40 + j)
        v = np.zeros(n, np.float32)
        for b in range(64):
            if (b + j) % 2 == 0:  # two records, both far into the bucket
                v[b * d + rng.integers(300, d, size=2)] = rng.standard_normal(2).astype(np.float32)
            else:
                v[b * d:(b + 1) * d] = rng.standard_normal(d).astype(np.float32)
        w, o, _, st = oracle_lib.encode(v, d, s, seed=5 + j)
        assert st == 0
        streams.append((w, o))
    base = _base(n, d, True)
    got, status = _run_multi(rows_exe, tmp_path, streams, n, d, s, False, base, grid=1, side=True)
    assert status == 0
    ref = base.copy()
    _, rst = oracle_lib.decode_accumulate(streams, n, d, s, ref)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("K", [3, 10])
def test_side_decoder_corrupt_stream(rows_exe, tmp_path, oracle_lib, K):
    """Bit flips in stream 1: the input is flagged, and every bucket no flip touched
    equals the oracle's sum, in later groups of the same CTA too (one CTA: its rings
    are reused after the malformed buckets)."""
    n, d, s = 40_000, 512, 4
    intact, streams = [], []
    for j in range(K):
        w, o, _, _ = oracle_lib.encode(W.small_normal(n, 70 + j), d, s, seed=j)
        intact.append((w, o))
        w2 = w.copy()
        if j == 1:
            _flip_bits(w2, o, np.random.default_rng(9))
        streams.append((w2, o))
    base = _base(n, d, True)
    got, status = _run_multi(rows_exe, tmp_path, streams, n, d, s, False, base, grid=1, side=True)
    assert status & 2
    ref = base.copy()
    oracle_lib.decode_accumulate(intact, n, d, s, ref)
    keep = np.ones(n, dtype=bool)
    flipped = streams[1][0] != intact[1][0]
    offs = intact[1][1]
    for b in range(offs.size - 1):
        w0, w1 = int(offs[b]) >> 5, (int(offs[b + 1]) + 31) >> 5
        if flipped[w0:w1].any():
            keep[b * d:min(n, (b + 1) * d)] = False
    assert keep.any() and not keep.all()
    assert np.array_equal(got[keep].view(np.uint32), ref[keep].view(np.uint32))


def _bucket_bits(words, offsets, b):
    """Bucket b's bits (MSB-first) as a numpy array of 0/1."""
    bits = np.unpackbits(words.astype(">u4").view(np.uint8))
    return bits[int(offsets[b]):int(offsets[b + 1])]


def _assemble(buckets):
    """A stream (words, offsets) from a list of per-bucket bit arrays."""
    offsets = np.zeros(len(buckets) + 1, np.uint64)
    offsets[1:] = np.cumsum([x.size for x in buckets])
    allbits = np.concatenate(buckets + [np.zeros((-int(offsets[-1])) % 32, np.uint8)])
    return np.packbits(allbits).view(">u4").astype(np.uint32), offsets


def test_side_decoder_overlong_bucket(rows_exe, tmp_path, oracle_lib):
    """A bucket whose records run past d (a well-formed bucket of 1024 coordinates in a
    stream of d = 512): flagged, and the codes it left beyond its row's last segment
    must not reach the buckets decoded after it by the same CTA."""
    n, d, s, K = 8 * 32 * 512, 512, 16, 3  # eight groups: four sets of two for one CTA
    streams = []
    for j in range(K):
        w, o, _, st = oracle_lib.encode(W.normal(n, 20 + j), d, s, seed=j)
        assert st == 0
        streams.append((w, o))
    long_w, long_o, _, _ = oracle_lib.encode(W.normal(1024, 5), 1024, s, seed=9)
    w1, o1 = streams[1]
    buckets = [_bucket_bits(w1, o1, b) for b in range(o1.size - 1)]
    buckets[3] = _bucket_bits(long_w, long_o, 0)
    streams[1] = _assemble(buckets)
    base = _base(n, d, True)
    got, status = _run_multi(rows_exe, tmp_path, streams, n, d, s, False, base, grid=1, side=True)
    assert status & 2
    intact = [streams[0], (w1, o1), streams[2]]
    ref = base.copy()
    oracle_lib.decode_accumulate(intact, n, d, s, ref)
    keep = np.ones(n, dtype=bool)
    keep[3 * d:4 * d] = False
    assert np.array_equal(got[keep].view(np.uint32), ref[keep].view(np.uint32))


# decode_sparse: buckets larger than the rows (d > 1024), decode and decode-accumulate
# of several streams in order; ragged last bucket, d not a multiple of four, long gaps
# (bit-serial records), s above the table's levels
SPARSE = [
    (60_001, 8192, 1, 1, False, "heavy_tailed_sparse"),
    (40_003, 3001, 16, 1, False, "layered"),
    (30_000, 2048, 300, 3, True, "normal"),
    (20_000, 4096, 4, 17, True, "small_normal"),
    (20_000, 2048, 1 << 20, 1, False, "normal"),  # levels past 16 bits (bit-serial)
    (65_536, 65_536, 256, 1, False, "normal"),    # one bucket (the small workload's shape)
]


@pytest.mark.parametrize("n,d,s,K,acc,kind", SPARSE, ids=["n%d-d%d-s%d-K%d-acc%d-%s" % c for c in SPARSE])
def test_large_bucket_decoder_matches_oracle(rows_exe, tmp_path, oracle_lib, n, d, s, K, acc, kind):
    streams = []
    for j in range(K):
        w, o, _, st = oracle_lib.encode(W.GENERATORS[kind](n, 90 + j), d, s, seed=j)
        assert st == 0
        streams.append((w, o))
    for j, (w, o) in enumerate(streams):
        np.concatenate([w, np.zeros(1, np.uint32)]).tofile(tmp_path / ("w%d.bin" % j))
        o.astype(np.uint64).tofile(tmp_path / ("o%d.bin" % j))
    base = _base(n, d, acc)
    base.tofile(tmp_path / "out_in.bin")
    np.array([n, d, s], np.uint64).tofile(tmp_path / "params.bin")
    r = subprocess.run([rows_exe, str(tmp_path), "1" if acc else "0", "2", "1", str(K), "0"],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-500:], r.stderr[-2000:])
    got, status = np.fromfile(tmp_path / "out.bin", np.float32), int(r.stdout.split()[-1])
    assert status == 0
    if acc:
        ref = base.copy()
        _, rst = oracle_lib.decode_accumulate(streams, n, d, s, ref)
    else:
        ref, rst = oracle_lib.decode(streams[0][0], streams[0][1], n, d, s)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("acc", [False, True])
def test_large_bucket_decoder_gap_boundaries(rows_exe, tmp_path, oracle_lib, acc):
    """Gaps at the edges of the long-record path (the gap-prefix table reads at most
    one 16-bit group): 63, 64, 2^15 - 1, 2^15, 2^16 - 1 take it; 2^16 and more take
    the bit-serial path.  Levels 15 (the level table's last) and 16 (past it)."""
    d, s = 70_000, 20
    gaps = [63, 64, 2 ** 15 - 1, 2 ** 15, 2 ** 16 - 1, 2 ** 16, 69_000]
    n = len(gaps) * d
    v = np.zeros(n, np.float32)
    for b, gap in enumerate(gaps):
        v[b * d] = 1.0  # the first record: gap 1
        v[b * d + gap] = -0.75 if b % 2 else 0.75
    words, offsets, _, st = oracle_lib.encode(v, d, s, seed=3)
    assert st == 0
    base = _base(n, d, acc)
    got, status = _run(rows_exe, tmp_path, words, offsets, n, d, s, acc, 2, 1, base)
    assert status == 0
    if acc:
        ref = base.copy()
        _, rst = oracle_lib.decode_accumulate([(words, offsets)], n, d, s, ref)
    else:
        ref, rst = oracle_lib.decode(words, offsets, n, d, s)
    assert rst == 0
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    if not acc:
        assert np.flatnonzero(ref).size == 2 * len(gaps)  # every far record decoded to a value

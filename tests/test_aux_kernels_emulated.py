"""The b-bit, error-feedback and mean kernels' exact source on the CPU block emulator.

qsgd_bbit.cu, qsgd_ef.cu and qsgd_mean.cu (their device code and grid-sizing helpers)
are compiled for the host under tests/emu/enc/block_emu.h and checked bit for bit
against the oracle:
- the b-bit encoder in its one-pass form (with and without the memory, both norm kinds)
  and its two-kernel form;
- the b-bit decoders in vector and scalar form, plain and accumulating;
- the pieces of the three-pass error feedback (e <- e + g; the residual after the
  Elias and the b-bit encodes);
- the division of the mean."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from emu_source import host_source
from gpu_common import check_norms
from quantized_gradient_compression_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_gradient_compression_b200", "csrc")
EMU = os.path.join(HERE, "emu", "enc")
CLOSE = "}  // namespace\n}  // namespace qsgd\n"


@pytest.fixture(scope="module")
def aux_exe(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("auxemu")
    src_dir = d / "pkg" / "csrc"
    src_dir.mkdir(parents=True)
    shutil.copytree(os.path.join(ROOT, "include"), d / "include")
    for h in ("qsgd_internal.h", "qsgd_limits.h"):
        shutil.copy(os.path.join(CSRC, h), src_dir / h)
    (src_dir / "qsgd_device.cuh").write_text(host_source(open(os.path.join(CSRC, "qsgd_device.cuh")).read()))
    parts = []
    for name, cut in (("qsgd_bbit.cu", "template <int B, bool kEF>\ncudaError_t launch_bbit_fast"),
                      ("qsgd_ef.cu", "}  // namespace\n\ncudaError_t launch_ef_add"),
                      ("qsgd_mean.cu", "}  // namespace\n\ncudaError_t launch_div")):
        text = open(os.path.join(CSRC, name)).read()
        parts.append(host_source(text[:text.index(cut)]) + CLOSE)
    (src_dir / "aux_emu.inc").write_text("\n".join(parts))
    exe = d / "aux_main"
    r = subprocess.run(["g++", "-O1", "-std=c++17", "-ffp-contract=off", "-pthread", "-I", EMU, "-I", str(src_dir),
                        os.path.join(EMU, "aux_main.cpp"), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    return str(exe)


def _params(tmp, n, d, bs, seed=0, nk=0, flag=0, cap=0):
    np.array([n, d, bs, seed, nk, flag, cap], np.uint64).tofile(tmp / "params.bin")


def _call(exe, tmp, op, grid=3):
    r = subprocess.run([exe, str(tmp), op, str(grid)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, (r.stdout[-500:], r.stderr[-2000:])
    return int(r.stdout.split()[-1])


def _bits(x):
    return np.asarray(x, np.float32).view(np.uint32)


# (n, d, b, memory, norm kind): one-pass shapes d = 128 V and two-kernel shapes
BB = [(20_003, 512, 4, False, 0), (10_000, 128, 2, True, 0), (9_001, 1024, 8, True, 1), (7_000, 100, 4, False, 0),
      (6_001, 384, 2, False, 1), (5_000, 256, 8, False, 0)]


@pytest.mark.parametrize("n,d,b,mem,nk", BB, ids=["n%d-d%d-b%d-m%d-nk%d" % c for c in BB])
def test_bbit_encoder(aux_exe, tmp_path, oracle_lib, n, d, b, mem, nk):
    g = W.layered(n, n % 31)
    e = W.normal(n, 3) * np.float32(0.05)
    _params(tmp_path, n, d, b, seed=9, nk=nk, flag=int(mem))
    g.tofile(tmp_path / "in.bin")
    if mem:
        e.tofile(tmp_path / "e.bin")
    st = _call(aux_exe, tmp_path, "bbit_enc")
    norms = np.fromfile(tmp_path / "norms.bin", np.float32)
    codes = np.fromfile(tmp_path / "codes.bin", np.uint32)
    if mem:
        own = oracle_lib.bbit_encode_ef(g, e, d, b, 9, max_norm=bool(nk))
        if nk:
            assert np.array_equal(_bits(norms), _bits(own[1]))
        else:
            check_norms(norms, own[1])
        r_codes, _, _, r_e = oracle_lib.bbit_encode_ef(g, e, d, b, 9, norms_in=norms)
        assert np.array_equal(_bits(np.fromfile(tmp_path / "e_out.bin", np.float32)), _bits(r_e))
    else:
        own = oracle_lib.bbit_encode(g, d, b, 9, norms_in=oracle_lib.maxnorms(g, d) if nk else None)
        if nk:
            assert np.array_equal(_bits(norms), _bits(own[1]))
        else:
            check_norms(norms, own[1])
        r_codes, _, _ = oracle_lib.bbit_encode(g, d, b, 9, norms_in=norms)
    assert st == own[2] and np.array_equal(codes, r_codes)


@pytest.mark.parametrize("n,d,b,vec,acc", [(20_000, 512, 4, 1, 0), (20_000, 512, 4, 1, 1), (7_001, 100, 2, 0, 1),
                                           (9_000, 128, 8, 0, 0), (10_001, 256, 2, 1, 1)])
def test_bbit_decoders(aux_exe, tmp_path, oracle_lib, n, d, b, vec, acc):
    codes, norms, _ = oracle_lib.bbit_encode(W.normal(n, 5), d, b, 2)
    base = W.normal(n, 6) * np.float32(0.01)
    base[::7] = np.float32(-0.0)
    _params(tmp_path, n, d, b, flag=vec)
    norms.tofile(tmp_path / "norms.bin")
    codes.tofile(tmp_path / "codes.bin")
    (base if acc else np.full(n, np.nan, np.float32)).tofile(tmp_path / "out.bin")
    assert _call(aux_exe, tmp_path, "bbit_acc" if acc else "bbit_dec") == 0
    got = np.fromfile(tmp_path / "out.bin", np.float32)
    if acc:
        ref = base.copy()
        oracle_lib.bbit_decode_accumulate([(norms, codes)], n, d, b, ref)
    else:
        ref, _ = oracle_lib.bbit_decode(norms, codes, n, d, b)
    assert np.array_equal(_bits(got), _bits(ref))


@pytest.mark.parametrize("n,vec", [(10_003, 1), (10_003, 0)])
def test_ef_add(aux_exe, tmp_path, n, vec):
    g = W.normal(n, 1)
    e = W.normal(n, 2) * np.float32(0.1)
    _params(tmp_path, n, 1, 1, flag=vec)
    g.tofile(tmp_path / "g.bin")
    e.tofile(tmp_path / "e.bin")
    _call(aux_exe, tmp_path, "ef_add")
    assert np.array_equal(_bits(np.fromfile(tmp_path / "e.bin", np.float32)), _bits(e + g))


@pytest.mark.parametrize("n,d,s", [(20_011, 100, 7), (9_000, 512, 16), (5_000, 6000, 2)])
def test_ef_residual_elias(aux_exe, tmp_path, oracle_lib, n, d, s):
    """The residual pass on the oracle's stream of p leaves the oracle's memory."""
    g = W.layered(n, 8)
    e = W.normal(n, 9) * np.float32(0.05)
    p = (e + g).astype(np.float32)
    words, offsets, _, _ = oracle_lib.encode(p, d, s, 4)
    _, _, _, _, r_e = oracle_lib.encode_ef(g, e, d, s, 4)
    _params(tmp_path, n, d, s, seed=4, cap=words.size)
    p.tofile(tmp_path / "e.bin")
    words.tofile(tmp_path / "words.bin")
    offsets.tofile(tmp_path / "offsets.bin")
    _call(aux_exe, tmp_path, "ef_res_elias")
    assert np.array_equal(_bits(np.fromfile(tmp_path / "e.bin", np.float32)), _bits(r_e))


@pytest.mark.parametrize("n,d,b", [(10_000, 100, 2), (9_001, 512, 8)])
def test_ef_residual_bbit(aux_exe, tmp_path, oracle_lib, n, d, b):
    g = W.normal(n, 10)
    e = W.normal(n, 11) * np.float32(0.05)
    p = (e + g).astype(np.float32)
    codes, norms, _ = oracle_lib.bbit_encode(p, d, b, 6)
    _, _, _, r_e = oracle_lib.bbit_encode_ef(g, e, d, b, 6)
    _params(tmp_path, n, d, b)
    p.tofile(tmp_path / "e.bin")
    norms.tofile(tmp_path / "norms.bin")
    codes.tofile(tmp_path / "codes.bin")
    _call(aux_exe, tmp_path, "ef_res_bbit")
    assert np.array_equal(_bits(np.fromfile(tmp_path / "e.bin", np.float32)), _bits(r_e))


@pytest.mark.parametrize("K,vec", [(3, 1), (7, 0), (1, 1)])
def test_mean_division(aux_exe, tmp_path, K, vec):
    x = W.normal(10_003, 12)
    x[5] = np.float32(-0.0)
    _params(tmp_path, x.size, 1, K, flag=vec)
    x.tofile(tmp_path / "out.bin")
    _call(aux_exe, tmp_path, "div")
    assert np.array_equal(_bits(np.fromfile(tmp_path / "out.bin", np.float32)), _bits(x / np.float32(K)))

"""CPU oracle for the QSGD codec -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding in ``quantized_gradient_compression_b200``) never imports it.

The arithmetic lives in ``qsgd_oracle.c`` (plain single-threaded C, fp32 ops in
source order, no FMA contraction).  This module only compiles it with gcc and
marshals numpy arrays through ctypes.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsgd_oracle.c")
_HDR = os.path.join(_HERE, "qsgd_oracle.h")
LIB_PATH = os.path.join(_HERE, "liboracle_qsgd.so")

CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra"]

ST_NONFINITE = 1
ST_BAD_STREAM = 2
ST_OVERFLOW = 8
ST_RANGE = 16

_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = LIB_PATH) -> str:
    """Compile the oracle with gcc.  Returns the path of the shared object."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(src), os.path.getmtime(_HDR))):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, "-I", os.path.dirname(src), src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, out)
    return out


def _declare(lib):
    u8p = ctypes.POINTER(ctypes.c_uint8)
    u32p = ctypes.POINTER(ctypes.c_uint32)
    u64p = ctypes.POINTER(ctypes.c_uint64)
    i32p = ctypes.POINTER(ctypes.c_int32)
    f32p = ctypes.POINTER(ctypes.c_float)
    c_u64, c_u32, c_int = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int
    sig = {
        "qo_philox4x32_10": (None, [u32p, u32p, u32p]),
        "qo_random_word": (c_u32, [c_u64, c_u64]),
        "qo_omega_len": (c_int, [c_u64]),
        "qo_omega_bits": (c_int, [c_u64, u8p]),
        "qo_omega_put": (c_int, [u32p, c_u64, u64p, c_u64]),
        "qo_omega_get": (c_int, [u32p, u64p, c_u64, u64p]),
        "qo_bucket_norm": (ctypes.c_float, [f32p, c_u64]),
        "qo_bucket_maxnorm": (ctypes.c_float, [f32p, c_u64]),
        "qo_quantize_bucket": (ctypes.c_float,
                               [f32p, c_u64, c_u64, c_u32, c_u64, f32p, i32p, u32p]),
        "qo_bucket_bit_bound": (c_u64, [c_u64, c_u32]),
        "qo_capacity_words": (c_u64, [c_u64, c_u64, c_u32]),
        "qo_encode": (c_int, [f32p, c_u64, c_u64, c_u32, c_u64, f32p, u32p, c_u64, u64p,
                              f32p, u32p]),
        "qo_encode_range": (c_int, [f32p, c_u64, c_u64, c_u32, c_u64, c_u64, c_u64, f32p, u32p, c_u64,
                                    u64p, f32p, u32p]),
        "qo_encode_bucket": (c_int, [f32p, c_u64, c_u64, c_u32, c_u64, f32p, u32p, c_u64, u64p,
                                     f32p, i32p, u32p]),
        "qo_decode_bucket": (c_int, [u32p, c_u64, c_u64, c_u64, c_u32, f32p, u32p]),
        "qo_decode": (c_int, [u32p, u64p, c_u64, c_u64, c_u32, f32p, u32p]),
        "qo_decode_levels": (c_int, [u32p, u64p, c_u64, c_u64, c_u32, i32p, f32p, u32p]),
        "qo_decode_accumulate": (c_int, [ctypes.POINTER(u32p), ctypes.POINTER(u64p), c_int,
                                         c_u64, c_u64, c_u32, f32p, u32p]),
        "qo_bbit_levels": (c_u32, [c_u32]),
        "qo_bbit_code_words": (c_u64, [c_u64, c_u32]),
        "qo_bbit_encode": (c_int, [f32p, c_u64, c_u64, c_u32, c_u64, f32p, f32p, u32p, u32p]),
        "qo_encode_ef": (c_int, [f32p, f32p, c_u64, c_u64, c_u32, c_u64, c_int, f32p, u32p, c_u64, u64p,
                                 f32p, u32p]),
        "qo_bbit_encode_ef": (c_int, [f32p, f32p, c_u64, c_u64, c_u32, c_u64, c_int, f32p, f32p, u32p, u32p]),
        "qo_bbit_decode": (c_int, [f32p, u32p, c_u64, c_u64, c_u32, f32p, u32p]),
        "qo_bbit_decode_accumulate": (c_int, [ctypes.POINTER(f32p), ctypes.POINTER(u32p), c_int,
                                              c_u64, c_u64, c_u32, f32p, u32p]),
        "qo_decode_mean": (c_int, [ctypes.POINTER(u32p), ctypes.POINTER(u64p), c_int,
                                   c_u64, c_u64, c_u32, f32p, u32p]),
        "qo_bbit_decode_mean": (c_int, [ctypes.POINTER(f32p), ctypes.POINTER(u32p), c_int,
                                        c_u64, c_u64, c_u32, f32p, u32p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    with _lock:
        if path is not None:
            return _declare(ctypes.CDLL(path))
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
        return _lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


class Oracle:
    """Thin numpy wrapper over one loaded oracle library."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    # --- primitives -------------------------------------------------------
    def philox(self, ctr, key):
        c = np.asarray(ctr, dtype=np.uint32).copy()
        k = np.asarray(key, dtype=np.uint32).copy()
        out = np.zeros(4, dtype=np.uint32)
        self.lib.qo_philox4x32_10(_ptr(c, ctypes.c_uint32), _ptr(k, ctypes.c_uint32),
                                  _ptr(out, ctypes.c_uint32))
        return out

    def random_word(self, seed: int, i: int) -> int:
        return int(self.lib.qo_random_word(seed, i))

    def omega_len(self, N: int) -> int:
        return int(self.lib.qo_omega_len(N))

    def omega_bits(self, N: int) -> str:
        buf = np.zeros(160, dtype=np.uint8)
        ln = self.lib.qo_omega_bits(N, _ptr(buf, ctypes.c_uint8))
        return "".join(str(int(b)) for b in buf[:ln])

    def omega_put_many(self, values) -> tuple[np.ndarray, int]:
        values = [int(x) for x in values]
        cap = sum(self.omega_len(x) for x in values) // 32 + 2
        words = np.zeros(cap, dtype=np.uint32)
        pos = ctypes.c_uint64(0)
        for x in values:
            rc = self.lib.qo_omega_put(_ptr(words, ctypes.c_uint32), cap, ctypes.byref(pos), x)
            assert rc == 0
        return words, pos.value

    def omega_get_many(self, words: np.ndarray, count: int, end_bit: int):
        pos = ctypes.c_uint64(0)
        out = []
        N = ctypes.c_uint64(0)
        for _ in range(count):
            rc = self.lib.qo_omega_get(_ptr(words, ctypes.c_uint32), ctypes.byref(pos), end_bit,
                                       ctypes.byref(N))
            if rc != 0:
                raise ValueError("omega_get failed")
            out.append(N.value)
        return out, pos.value

    def bucket_norm(self, v: np.ndarray) -> np.float32:
        v = np.ascontiguousarray(v, dtype=np.float32)
        return np.float32(self.lib.qo_bucket_norm(_ptr(v, ctypes.c_float), v.size))

    def bucket_maxnorm(self, v: np.ndarray) -> np.float32:
        v = np.ascontiguousarray(v, dtype=np.float32)
        if v.size == 0:
            return np.float32(0.0)
        return np.float32(self.lib.qo_bucket_maxnorm(_ptr(v, ctypes.c_float), v.size))

    def maxnorms(self, v: np.ndarray, d: int) -> np.ndarray:
        """The max-norm of every bucket: norms_in for the QSGDinf variant."""
        v = np.ascontiguousarray(v, dtype=np.float32)
        nb = (v.size + d - 1) // d
        return np.array([self.bucket_maxnorm(v[b * d:(b + 1) * d]) for b in range(nb)], dtype=np.float32)

    def capacity_words(self, n: int, d: int, s: int) -> int:
        return int(self.lib.qo_capacity_words(n, d, s))

    def bucket_bit_bound(self, m: int, s: int) -> int:
        return int(self.lib.qo_bucket_bit_bound(m, s))

    # --- whole-vector operations -----------------------------------------
    def quantize(self, v: np.ndarray, d: int, s: int, seed: int, norms_in=None):
        """Signed levels (int32[n]) and sent norms (float32[nb]) of every bucket."""
        v = np.ascontiguousarray(v, dtype=np.float32)
        n = v.size
        nb = (n + d - 1) // d
        levels = np.zeros(max(n, 1), dtype=np.int32)
        norms = np.zeros(max(nb, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        for b in range(nb):
            base = b * d
            m = min(d, n - base)
            nin = None
            if norms_in is not None:
                nin = np.asarray([norms_in[b]], dtype=np.float32)
            vb = v[base:base + m]
            norms[b] = self.lib.qo_quantize_bucket(
                _ptr(vb, ctypes.c_float), m, base, s, seed,
                _ptr(nin, ctypes.c_float) if nin is not None else None,
                _ptr(levels[base:base + m], ctypes.c_int32), ctypes.byref(st))
        return levels[:n], norms[:nb], st.value

    def encode(self, v: np.ndarray, d: int, s: int, seed: int, norms_in=None):
        """Returns (words uint32[ceil(bits/32)], offsets uint64[nb+1], norms, status)."""
        v = np.ascontiguousarray(v, dtype=np.float32)
        n = v.size
        nb = (n + d - 1) // d
        cap = self.capacity_words(n, d, s)
        words = np.zeros(max(cap, 1), dtype=np.uint32)
        offsets = np.zeros(nb + 1, dtype=np.uint64)
        norms = np.zeros(max(nb, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        nin = None
        if norms_in is not None:
            nin = np.ascontiguousarray(norms_in, dtype=np.float32)
            assert nin.size == nb
        rc = self.lib.qo_encode(_ptr(v, ctypes.c_float) if n else None, n, d, s, seed,
                                _ptr(nin, ctypes.c_float) if nin is not None else None,
                                _ptr(words, ctypes.c_uint32), cap, _ptr(offsets, ctypes.c_uint64),
                                _ptr(norms, ctypes.c_float), ctypes.byref(st))
        if rc != 0:
            raise RuntimeError("oracle encode failed (status %d)" % st.value)
        nwords = (int(offsets[nb]) + 31) // 32
        return words[:nwords].copy(), offsets, norms[:nb], st.value

    def encode_range(self, v: np.ndarray, d: int, s: int, seed: int, b0: int, b1: int, norms_in=None):
        """Buckets [b0, b1) of v as a standalone stream: (words, offsets relative to the
        slice, norms, status); the bits of those buckets in encode()'s stream."""
        assert v.dtype == np.float32 and v.flags["C_CONTIGUOUS"]
        n = v.size
        nb = (n + d - 1) // d
        assert 0 <= b0 <= b1 <= nb
        m = min(n, b1 * d) - b0 * d
        cap = (32 * (b1 - b0) + m * (2 + self.omega_len(s)) + 31) // 32 + 1
        words = np.zeros(cap, dtype=np.uint32)
        offsets = np.zeros(b1 - b0 + 1, dtype=np.uint64)
        norms = np.zeros(max(b1 - b0, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        nin = None
        if norms_in is not None:
            nin = np.ascontiguousarray(norms_in, dtype=np.float32)
            assert nin.size == b1 - b0
        rc = self.lib.qo_encode_range(_ptr(v, ctypes.c_float), n, d, s, seed, b0, b1,
                                      _ptr(nin, ctypes.c_float) if nin is not None else None,
                                      _ptr(words, ctypes.c_uint32), cap, _ptr(offsets, ctypes.c_uint64),
                                      _ptr(norms, ctypes.c_float), ctypes.byref(st))
        if rc != 0:
            raise RuntimeError("oracle encode_range failed (status %d)" % st.value)
        nwords = (int(offsets[-1]) + 31) // 32
        return words[:nwords].copy(), offsets, norms[:b1 - b0], st.value

    def encode_bucket(self, vb: np.ndarray, base: int, s: int, seed: int, norm_in=None):
        """One bucket at global index `base` as a standalone bit string (words, nbits)."""
        vb = np.ascontiguousarray(vb, dtype=np.float32)
        m = vb.size
        cap = (32 + m * (2 + self.omega_len(s))) // 32 + 2
        words = np.zeros(cap, dtype=np.uint32)
        levels = np.zeros(max(m, 1), dtype=np.int32)
        pos = ctypes.c_uint64(0)
        st = ctypes.c_uint32(0)
        nin = None if norm_in is None else np.asarray([norm_in], dtype=np.float32)
        norm = np.zeros(1, dtype=np.float32)
        rc = self.lib.qo_encode_bucket(_ptr(vb, ctypes.c_float), m, base, s, seed,
                                       _ptr(nin, ctypes.c_float) if nin is not None else None,
                                       _ptr(words, ctypes.c_uint32), cap, ctypes.byref(pos),
                                       _ptr(norm, ctypes.c_float), _ptr(levels, ctypes.c_int32),
                                       ctypes.byref(st))
        assert rc == 0
        return words, pos.value, st.value

    def decode_bucket(self, words: np.ndarray, begin: int, end: int, m: int, s: int):
        words = np.ascontiguousarray(words, dtype=np.uint32)
        out = np.zeros(max(m, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        rc = self.lib.qo_decode_bucket(_ptr(words, ctypes.c_uint32), begin, end, m, s,
                                       _ptr(out, ctypes.c_float), ctypes.byref(st))
        assert rc == 0
        return out[:m], st.value

    def decode(self, words: np.ndarray, offsets: np.ndarray, n: int, d: int, s: int):
        words = np.ascontiguousarray(words, dtype=np.uint32)
        if words.size == 0:
            words = np.zeros(1, dtype=np.uint32)
        offsets = np.ascontiguousarray(offsets, dtype=np.uint64)
        out = np.zeros(max(n, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        rc = self.lib.qo_decode(_ptr(words, ctypes.c_uint32), _ptr(offsets, ctypes.c_uint64), n,
                                d, s, _ptr(out, ctypes.c_float), ctypes.byref(st))
        assert rc == 0
        return out[:n], st.value

    def decode_levels(self, words: np.ndarray, offsets: np.ndarray, n: int, d: int, s: int):
        words = np.ascontiguousarray(words, dtype=np.uint32)
        if words.size == 0:
            words = np.zeros(1, dtype=np.uint32)
        offsets = np.ascontiguousarray(offsets, dtype=np.uint64)
        nb = (n + d - 1) // d
        levels = np.zeros(max(n, 1), dtype=np.int32)
        norms = np.zeros(max(nb, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        rc = self.lib.qo_decode_levels(_ptr(words, ctypes.c_uint32),
                                       _ptr(offsets, ctypes.c_uint64), n, d, s,
                                       _ptr(levels, ctypes.c_int32), _ptr(norms, ctypes.c_float),
                                       ctypes.byref(st))
        assert rc == 0
        return levels[:n], norms[:nb], st.value

    def decode_accumulate(self, streams, n: int, d: int, s: int, out: np.ndarray):
        """streams: list of (words, offsets).  out is updated in place and returned."""
        K = len(streams)
        ws = [np.ascontiguousarray(w if w.size else np.zeros(1, np.uint32), dtype=np.uint32)
              for w, _ in streams]
        os_ = [np.ascontiguousarray(o, dtype=np.uint64) for _, o in streams]
        u32p = ctypes.POINTER(ctypes.c_uint32)
        u64p = ctypes.POINTER(ctypes.c_uint64)
        wp = (u32p * K)(*[_ptr(w, ctypes.c_uint32) for w in ws])
        op = (u64p * K)(*[_ptr(o, ctypes.c_uint64) for o in os_])
        assert out.dtype == np.float32 and out.flags["C_CONTIGUOUS"] and out.size == n
        st = ctypes.c_uint32(0)
        buf = out if n else np.zeros(1, np.float32)
        rc = self.lib.qo_decode_accumulate(wp, op, K, n, d, s, _ptr(buf, ctypes.c_float),
                                           ctypes.byref(st))
        assert rc == 0
        return out, st.value


    def decode_mean(self, streams, n: int, d: int, s: int):
        """Mean of the K decoded streams (list of (words, offsets)): (sum from +0) / K."""
        K = len(streams)
        ws = [np.ascontiguousarray(w if w.size else np.zeros(1, np.uint32), dtype=np.uint32)
              for w, _ in streams]
        os_ = [np.ascontiguousarray(o, dtype=np.uint64) for _, o in streams]
        u32p = ctypes.POINTER(ctypes.c_uint32)
        u64p = ctypes.POINTER(ctypes.c_uint64)
        wp = (u32p * K)(*[_ptr(w, ctypes.c_uint32) for w in ws])
        op = (u64p * K)(*[_ptr(o, ctypes.c_uint64) for o in os_])
        out = np.zeros(max(n, 1), np.float32)
        st = ctypes.c_uint32(0)
        rc = self.lib.qo_decode_mean(wp, op, K, n, d, s, _ptr(out, ctypes.c_float), ctypes.byref(st))
        assert rc == 0
        return out[:n], st.value

    # ---- fixed-width b-bit variant ----------------------------------------------
    def bbit_levels(self, b: int) -> int:
        return int(self.lib.qo_bbit_levels(b))

    def bbit_code_words(self, n: int, b: int) -> int:
        return int(self.lib.qo_bbit_code_words(n, b))

    def bbit_encode(self, v: np.ndarray, d: int, b: int, seed: int, norms_in=None):
        """Returns (codes uint32[ceil(n*b/32)], norms float32[nb], status)."""
        v = np.ascontiguousarray(v, dtype=np.float32)
        n = v.size
        nb = (n + d - 1) // d
        codes = np.zeros(max(self.bbit_code_words(n, b), 1), dtype=np.uint32)
        norms = np.zeros(max(nb, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        nin = None
        if norms_in is not None:
            nin = np.ascontiguousarray(norms_in, dtype=np.float32)
            assert nin.size == nb
        vv = v if n else np.zeros(1, np.float32)
        rc = self.lib.qo_bbit_encode(_ptr(vv, ctypes.c_float), n, d, b, seed,
                                     _ptr(nin, ctypes.c_float) if nin is not None else None,
                                     _ptr(norms, ctypes.c_float), _ptr(codes, ctypes.c_uint32),
                                     ctypes.byref(st))
        if rc != 0:
            raise ValueError("oracle b-bit encode rejected b=%d d=%d" % (b, d))
        return codes[:self.bbit_code_words(n, b)].copy(), norms[:nb].copy(), st.value

    # --- error feedback ("Sparsified SGD with Memory") ----------------------
    def encode_ef(self, g: np.ndarray, e: np.ndarray, d: int, s: int, seed: int, max_norm: bool = False,
                  norms_in=None):
        """p = e + g is encoded; returns (words, offsets, norms, status, e_new) with
        e_new = p - Q(p) (p where no record was sent).  e is not modified."""
        g = np.ascontiguousarray(g, dtype=np.float32)
        e_new = np.array(e, dtype=np.float32, copy=True)
        n = g.size
        assert e_new.size == n
        nb = (n + d - 1) // d
        cap = self.capacity_words(n, d, s)
        words = np.zeros(max(cap, 1), dtype=np.uint32)
        offsets = np.zeros(nb + 1, dtype=np.uint64)
        norms = np.zeros(max(nb, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        nin = None if norms_in is None else np.ascontiguousarray(norms_in, dtype=np.float32)
        gg = g if n else np.zeros(1, np.float32)
        ee = e_new if n else np.zeros(1, np.float32)
        rc = self.lib.qo_encode_ef(_ptr(gg, ctypes.c_float), _ptr(ee, ctypes.c_float), n, d, s, seed,
                                   int(bool(max_norm)), _ptr(nin, ctypes.c_float) if nin is not None else None,
                                   _ptr(words, ctypes.c_uint32), cap, _ptr(offsets, ctypes.c_uint64),
                                   _ptr(norms, ctypes.c_float), ctypes.byref(st))
        if rc != 0:
            raise RuntimeError("oracle error-feedback encode failed (status %d)" % st.value)
        nwords = (int(offsets[nb]) + 31) // 32
        return words[:nwords].copy(), offsets, norms[:nb].copy(), st.value, e_new[:n]

    def bbit_encode_ef(self, g: np.ndarray, e: np.ndarray, d: int, b: int, seed: int, max_norm: bool = False,
                       norms_in=None):
        """b-bit codes of p = e + g; returns (codes, norms, status, e_new)."""
        g = np.ascontiguousarray(g, dtype=np.float32)
        e_new = np.array(e, dtype=np.float32, copy=True)
        n = g.size
        assert e_new.size == n
        nb = (n + d - 1) // d
        codes = np.zeros(max(self.bbit_code_words(n, b), 1), dtype=np.uint32)
        norms = np.zeros(max(nb, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        nin = None if norms_in is None else np.ascontiguousarray(norms_in, dtype=np.float32)
        gg = g if n else np.zeros(1, np.float32)
        ee = e_new if n else np.zeros(1, np.float32)
        rc = self.lib.qo_bbit_encode_ef(_ptr(gg, ctypes.c_float), _ptr(ee, ctypes.c_float), n, d, b, seed,
                                        int(bool(max_norm)),
                                        _ptr(nin, ctypes.c_float) if nin is not None else None,
                                        _ptr(norms, ctypes.c_float), _ptr(codes, ctypes.c_uint32),
                                        ctypes.byref(st))
        if rc != 0:
            raise ValueError("oracle b-bit error-feedback encode rejected b=%d d=%d" % (b, d))
        return codes[:self.bbit_code_words(n, b)].copy(), norms[:nb].copy(), st.value, e_new[:n]

    def bbit_decode(self, norms: np.ndarray, codes: np.ndarray, n: int, d: int, b: int):
        norms = np.ascontiguousarray(norms, dtype=np.float32)
        codes = np.ascontiguousarray(codes, dtype=np.uint32)
        if codes.size == 0:
            codes = np.zeros(1, np.uint32)
        if norms.size == 0:
            norms = np.zeros(1, np.float32)
        out = np.zeros(max(n, 1), dtype=np.float32)
        st = ctypes.c_uint32(0)
        rc = self.lib.qo_bbit_decode(_ptr(norms, ctypes.c_float), _ptr(codes, ctypes.c_uint32), n, d, b,
                                     _ptr(out, ctypes.c_float), ctypes.byref(st))
        assert rc == 0
        return out[:n], st.value

    def bbit_decode_accumulate(self, streams, n: int, d: int, b: int, out: np.ndarray):
        """streams: list of (norms, codes).  out is updated in place and returned."""
        K = len(streams)
        ns = [np.ascontiguousarray(x if x.size else np.zeros(1, np.float32), dtype=np.float32)
              for x, _ in streams]
        cs = [np.ascontiguousarray(c if c.size else np.zeros(1, np.uint32), dtype=np.uint32)
              for _, c in streams]
        f32p = ctypes.POINTER(ctypes.c_float)
        u32p = ctypes.POINTER(ctypes.c_uint32)
        npp = (f32p * K)(*[_ptr(x, ctypes.c_float) for x in ns])
        cpp = (u32p * K)(*[_ptr(c, ctypes.c_uint32) for c in cs])
        assert out.dtype == np.float32 and out.flags["C_CONTIGUOUS"] and out.size == n
        st = ctypes.c_uint32(0)
        buf = out if n else np.zeros(1, np.float32)
        rc = self.lib.qo_bbit_decode_accumulate(npp, cpp, K, n, d, b, _ptr(buf, ctypes.c_float),
                                                ctypes.byref(st))
        assert rc == 0
        return out, st.value


    def bbit_decode_mean(self, streams, n: int, d: int, b: int):
        """Mean of the K decoded b-bit streams (list of (norms, codes))."""
        K = len(streams)
        ns = [np.ascontiguousarray(x if x.size else np.zeros(1, np.float32), dtype=np.float32)
              for x, _ in streams]
        cs = [np.ascontiguousarray(c if c.size else np.zeros(1, np.uint32), dtype=np.uint32)
              for _, c in streams]
        f32p = ctypes.POINTER(ctypes.c_float)
        u32p = ctypes.POINTER(ctypes.c_uint32)
        npp = (f32p * K)(*[_ptr(x, ctypes.c_float) for x in ns])
        cpp = (u32p * K)(*[_ptr(c, ctypes.c_uint32) for c in cs])
        out = np.zeros(max(n, 1), np.float32)
        st = ctypes.c_uint32(0)
        rc = self.lib.qo_bbit_decode_mean(npp, cpp, K, n, d, b, _ptr(out, ctypes.c_float), ctypes.byref(st))
        assert rc == 0
        return out[:n], st.value


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default

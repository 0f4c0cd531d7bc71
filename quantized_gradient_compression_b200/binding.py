"""ctypes binding of the QSGD C ABI (include/qsgd.h): argument marshalling only.

The entry points keep the C names and take raw device pointers (ints), sizes and a
CUDA stream handle.  Every step of the codec runs in the CUDA library; there is
no CPU fallback: importing this module fails if ``libqsgd_b200.so`` is missing.

The torch helpers at the bottom (``encode``, ``decode``, ``decode_accumulate``)
only allocate device memory with torch and pass pointers and torch's current
stream through.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqsgd_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "the QSGD CUDA library %s is not built; run "
        "`python -m quantized_gradient_compression_b200.build` (nvcc, sm_100a)" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

QSGD_OK = 0
QSGD_ERR_ARG = 1
QSGD_ERR_CAPACITY = 2
QSGD_ERR_CUDA = 3
QSGD_ERR_WORKSPACE = 4
QSGD_ERR_STATIC_LIMIT = 5

QSGD_ST_NONFINITE = 1
QSGD_ST_BAD_STREAM = 2
QSGD_ST_LOOKBACK_TIMEOUT = 4
QSGD_ST_OVERFLOW = 8
QSGD_ST_RANGE = 16

QSGD_NORM_L2 = 0
QSGD_NORM_MAX = 1

_u64, _u32, _int, _sz, _vp = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p

_SIGS = {
    "qsgd_num_buckets": (_u64, [_u64, _u32]),
    "qsgd_max_encoded_words": (_u64, [_u64, _u32, _u32]),
    "qsgd_encode_workspace_bytes": (_sz, [_u64, _u32, _u32]),
    "qsgd_workspace_init": (_int, [_vp, _sz, _vp]),
    "qsgd_encode": (_int, [_vp, _u64, _u32, _u32, _u64, _vp, _u64, _vp, _vp, _sz, _vp, _vp]),
    "qsgd_encode_ex": (_int, [_vp, _u64, _u32, _u32, _u64, _u32, _vp, _u64, _vp, _vp, _sz, _vp, _vp]),
    "qsgd_encode_ef": (_int, [_vp, _vp, _u64, _u32, _u32, _u64, _u32, _vp, _u64, _vp, _vp, _sz, _vp, _vp]),
    "qsgd_decode": (_int, [_vp, _u64, _vp, _u64, _u32, _u32, _vp, _vp, _vp]),
    "qsgd_decode_accumulate": (_int, [ctypes.POINTER(_vp), ctypes.POINTER(_u64), ctypes.POINTER(_vp),
                                      _int, _u64, _u32, _u32, _vp, _vp, _vp]),
    "qsgd_decode_mean": (_int, [ctypes.POINTER(_vp), ctypes.POINTER(_u64), ctypes.POINTER(_vp),
                                _int, _u64, _u32, _u32, _vp, _vp, _vp]),
    "qsgd_encode_static_ws": (_int, [_vp, _u64, _u32, _u32, _u64, _vp, _u64, _vp, _vp, _vp]),
    "qsgd_static_workspace_limit": (_sz, []),
    "qsgd_bbit_code_words": (_u64, [_u64, _u32]),
    "qsgd_bbit_encode": (_int, [_vp, _u64, _u32, _u32, _u64, _vp, _vp, _vp, _vp]),
    "qsgd_bbit_encode_ex": (_int, [_vp, _u64, _u32, _u32, _u64, _u32, _vp, _vp, _vp, _vp]),
    "qsgd_bbit_encode_ef": (_int, [_vp, _vp, _u64, _u32, _u32, _u64, _u32, _vp, _vp, _vp, _vp]),
    "qsgd_bbit_decode": (_int, [_vp, _vp, _u64, _u32, _u32, _vp, _vp, _vp]),
    "qsgd_bbit_decode_accumulate": (_int, [ctypes.POINTER(_vp), ctypes.POINTER(_vp), _int, _u64, _u32, _u32,
                                           _vp, _vp, _vp]),
    "qsgd_bbit_decode_mean": (_int, [ctypes.POINTER(_vp), ctypes.POINTER(_vp), _int, _u64, _u32, _u32,
                                     _vp, _vp, _vp]),
    "qsgd_error_string": (ctypes.c_char_p, [_int]),
    "qsgd_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


class QsgdError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__("%s: %s (code %d)" % (where, qsgd_error_string(code), code))
        self.code = code


def _check(code: int, where: str) -> int:
    if code != QSGD_OK:
        raise QsgdError(code, where)
    return code


# --- C entry points (same names, same argument order) -----------------------

def qsgd_num_buckets(n: int, d: int) -> int:
    return int(_lib.qsgd_num_buckets(n, d))


def qsgd_max_encoded_words(n: int, d: int, s: int) -> int:
    return int(_lib.qsgd_max_encoded_words(n, d, s))


def qsgd_encode_workspace_bytes(n: int, d: int, s: int) -> int:
    return int(_lib.qsgd_encode_workspace_bytes(n, d, s))


def qsgd_workspace_init(d_ws: int, ws_bytes: int, stream: int) -> int:
    return int(_lib.qsgd_workspace_init(d_ws, ws_bytes, stream))


def qsgd_encode(d_in: int, n: int, d: int, s: int, seed: int, d_words: int, words_capacity: int,
                d_offsets: int, d_ws: int, ws_bytes: int, d_status: int, stream: int) -> int:
    return int(_lib.qsgd_encode(d_in, n, d, s, seed & 0xFFFFFFFFFFFFFFFF, d_words, words_capacity,
                                d_offsets, d_ws, ws_bytes, d_status, stream))


def qsgd_encode_ex(d_in: int, n: int, d: int, s: int, seed: int, norm_kind: int, d_words: int,
                   words_capacity: int, d_offsets: int, d_ws: int, ws_bytes: int, d_status: int, stream: int) -> int:
    return int(_lib.qsgd_encode_ex(d_in, n, d, s, seed & 0xFFFFFFFFFFFFFFFF, norm_kind, d_words, words_capacity,
                                   d_offsets, d_ws, ws_bytes, d_status, stream))


def qsgd_encode_ef(d_g: int, d_e: int, n: int, d: int, s: int, seed: int, norm_kind: int, d_words: int,
                   words_capacity: int, d_offsets: int, d_ws: int, ws_bytes: int, d_status: int, stream: int) -> int:
    return int(_lib.qsgd_encode_ef(d_g, d_e, n, d, s, seed & 0xFFFFFFFFFFFFFFFF, norm_kind, d_words, words_capacity,
                                   d_offsets, d_ws, ws_bytes, d_status, stream))


def qsgd_decode(d_words: int, num_words: int, d_offsets: int, n: int, d: int, s: int, d_out: int,
                d_status: int, stream: int) -> int:
    return int(_lib.qsgd_decode(d_words, num_words, d_offsets, n, d, s, d_out, d_status, stream))


def qsgd_decode_accumulate(h_words, h_num_words, h_offsets, K: int, n: int, d: int, s: int,
                           d_out: int, d_status: int, stream: int) -> int:
    w = (_vp * K)(*h_words)
    nw = (_u64 * K)(*h_num_words)
    o = (_vp * K)(*h_offsets)
    return int(_lib.qsgd_decode_accumulate(w, nw, o, K, n, d, s, d_out, d_status, stream))


def qsgd_decode_mean(h_words, h_num_words, h_offsets, K: int, n: int, d: int, s: int,
                     d_out: int, d_status: int, stream: int) -> int:
    w = (_vp * K)(*h_words)
    nw = (_u64 * K)(*h_num_words)
    o = (_vp * K)(*h_offsets)
    return int(_lib.qsgd_decode_mean(w, nw, o, K, n, d, s, d_out, d_status, stream))


def qsgd_encode_static_ws(d_in: int, n: int, d: int, s: int, seed: int, d_words: int, words_capacity: int,
                          d_offsets: int, d_status: int, stream: int) -> int:
    """qsgd_encode without a caller workspace (for callers that cannot allocate)."""
    return int(_lib.qsgd_encode_static_ws(d_in, n, d, s, seed & 0xFFFFFFFFFFFFFFFF, d_words, words_capacity,
                                          d_offsets, d_status, stream))


def qsgd_static_workspace_limit() -> int:
    return int(_lib.qsgd_static_workspace_limit())


def qsgd_bbit_code_words(n: int, b: int) -> int:
    return int(_lib.qsgd_bbit_code_words(n, b))


def qsgd_bbit_encode(d_in: int, n: int, d: int, b: int, seed: int, d_norms: int, d_codes: int, d_status: int,
                     stream: int) -> int:
    return int(_lib.qsgd_bbit_encode(d_in, n, d, b, seed & 0xFFFFFFFFFFFFFFFF, d_norms, d_codes, d_status, stream))


def qsgd_bbit_encode_ex(d_in: int, n: int, d: int, b: int, seed: int, norm_kind: int, d_norms: int, d_codes: int,
                        d_status: int, stream: int) -> int:
    return int(_lib.qsgd_bbit_encode_ex(d_in, n, d, b, seed & 0xFFFFFFFFFFFFFFFF, norm_kind, d_norms, d_codes,
                                        d_status, stream))


def qsgd_bbit_encode_ef(d_g: int, d_e: int, n: int, d: int, b: int, seed: int, norm_kind: int, d_norms: int,
                        d_codes: int, d_status: int, stream: int) -> int:
    return int(_lib.qsgd_bbit_encode_ef(d_g, d_e, n, d, b, seed & 0xFFFFFFFFFFFFFFFF, norm_kind, d_norms, d_codes,
                                        d_status, stream))


def qsgd_bbit_decode(d_norms: int, d_codes: int, n: int, d: int, b: int, d_out: int, d_status: int,
                     stream: int) -> int:
    return int(_lib.qsgd_bbit_decode(d_norms, d_codes, n, d, b, d_out, d_status, stream))


def qsgd_bbit_decode_accumulate(h_norms, h_codes, K: int, n: int, d: int, b: int, d_out: int, d_status: int,
                                stream: int) -> int:
    nn = (_vp * K)(*h_norms)
    cc = (_vp * K)(*h_codes)
    return int(_lib.qsgd_bbit_decode_accumulate(nn, cc, K, n, d, b, d_out, d_status, stream))


def qsgd_bbit_decode_mean(h_norms, h_codes, K: int, n: int, d: int, b: int, d_out: int, d_status: int,
                          stream: int) -> int:
    nn = (_vp * K)(*h_norms)
    cc = (_vp * K)(*h_codes)
    return int(_lib.qsgd_bbit_decode_mean(nn, cc, K, n, d, b, d_out, d_status, stream))


def qsgd_error_string(code: int) -> str:
    return _lib.qsgd_error_string(code).decode()


def qsgd_version() -> str:
    return _lib.qsgd_version().decode()


# --- torch helpers: device memory and the current stream, nothing else -------

@dataclass
class Encoded:
    words: "object"    # torch.int32 tensor on the device (uint32 bit patterns)
    offsets: "object"  # torch.int64 tensor [nb+1] (uint64 bit offsets)
    n: int
    d: int
    s: int
    seed: int
    status: "object"   # torch.int32 tensor [1]

    @property
    def num_words(self) -> int:
        return int(self.words.numel())


_workspaces = {}


def _torch():
    import torch

    return torch


def workspace(n: int, d: int, s: int, device, stream_handle: int):
    """A zero-initialised workspace tensor shared by calls on one (device, stream)."""
    torch = _torch()
    need = qsgd_encode_workspace_bytes(n, d, s)
    key = (str(device), stream_handle)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def encode(x, d: int, s: int, seed: int, words=None, offsets=None, status=None,
           norm_kind: int = QSGD_NORM_L2) -> Encoded:
    torch = _torch()
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    n = x.numel()
    nb = qsgd_num_buckets(n, d)
    cap = qsgd_max_encoded_words(n, d, s)
    dev = x.device
    stream = torch.cuda.current_stream(dev).cuda_stream
    if words is None:
        words = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    if offsets is None:
        offsets = torch.empty(nb + 1, dtype=torch.int64, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = workspace(n, d, s, dev, stream)
    _check(qsgd_encode_ex(x.data_ptr(), n, d, s, seed, norm_kind, words.data_ptr(), words.numel(),
                          offsets.data_ptr(), ws.data_ptr(), ws.numel(), status.data_ptr(), stream), "qsgd_encode_ex")
    return Encoded(words, offsets, n, d, s, seed, status)


def encode_ef(g, e, d: int, s: int, seed: int, words=None, offsets=None, status=None,
              norm_kind: int = QSGD_NORM_L2) -> Encoded:
    """Error feedback: encodes p = e + g and leaves p minus its decoded value in e."""
    torch = _torch()
    for t in (g, e):
        assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    n = g.numel()
    assert e.numel() == n
    nb = qsgd_num_buckets(n, d)
    cap = qsgd_max_encoded_words(n, d, s)
    dev = g.device
    stream = torch.cuda.current_stream(dev).cuda_stream
    if words is None:
        words = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    if offsets is None:
        offsets = torch.empty(nb + 1, dtype=torch.int64, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = workspace(n, d, s, dev, stream)
    _check(qsgd_encode_ef(g.data_ptr(), e.data_ptr(), n, d, s, seed, norm_kind, words.data_ptr(), words.numel(),
                          offsets.data_ptr(), ws.data_ptr(), ws.numel(), status.data_ptr(), stream), "qsgd_encode_ef")
    return Encoded(words, offsets, n, d, s, seed, status)


def decode(enc: Encoded, out=None, status=None):
    torch = _torch()
    dev = enc.words.device
    if out is None:
        out = torch.empty(enc.n, dtype=torch.float32, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    _check(qsgd_decode(enc.words.data_ptr(), enc.num_words, enc.offsets.data_ptr(), enc.n, enc.d, enc.s,
                       out.data_ptr(), status.data_ptr(), stream), "qsgd_decode")
    return out, status


def decode_accumulate(encs, out, status=None):
    torch = _torch()
    e0 = encs[0]
    dev = out.device
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    _check(qsgd_decode_accumulate([e.words.data_ptr() for e in encs], [e.num_words for e in encs],
                                  [e.offsets.data_ptr() for e in encs], len(encs), e0.n, e0.d, e0.s,
                                  out.data_ptr(), status.data_ptr(), stream), "qsgd_decode_accumulate")
    return out, status


# --- fixed-width b-bit variant -------------------------------------------------

@dataclass
class BbitEncoded:
    norms: "object"   # torch.float32 tensor [nb]
    codes: "object"   # torch.int32 tensor [qsgd_bbit_code_words(n, b)] (uint32 bit patterns)
    n: int
    d: int
    b: int
    seed: int
    status: "object"  # torch.int32 tensor [1]


def bbit_encode(x, d: int, b: int, seed: int, norms=None, codes=None, status=None,
                norm_kind: int = QSGD_NORM_L2) -> BbitEncoded:
    torch = _torch()
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    n = x.numel()
    dev = x.device
    stream = torch.cuda.current_stream(dev).cuda_stream
    if norms is None:
        norms = torch.empty(max(qsgd_num_buckets(n, d), 1), dtype=torch.float32, device=dev)
    if codes is None:
        codes = torch.empty(max(qsgd_bbit_code_words(n, b), 1), dtype=torch.int32, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    _check(qsgd_bbit_encode_ex(x.data_ptr(), n, d, b, seed, norm_kind, norms.data_ptr(), codes.data_ptr(),
                               status.data_ptr(), stream), "qsgd_bbit_encode_ex")
    return BbitEncoded(norms, codes, n, d, b, seed, status)


def bbit_encode_ef(g, e, d: int, b: int, seed: int, norms=None, codes=None, status=None,
                   norm_kind: int = QSGD_NORM_L2) -> BbitEncoded:
    """Error feedback: codes p = e + g and leaves p minus its decoded value in e."""
    torch = _torch()
    for t in (g, e):
        assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    n = g.numel()
    assert e.numel() == n
    dev = g.device
    stream = torch.cuda.current_stream(dev).cuda_stream
    if norms is None:
        norms = torch.empty(max(qsgd_num_buckets(n, d), 1), dtype=torch.float32, device=dev)
    if codes is None:
        codes = torch.empty(max(qsgd_bbit_code_words(n, b), 1), dtype=torch.int32, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    _check(qsgd_bbit_encode_ef(g.data_ptr(), e.data_ptr(), n, d, b, seed, norm_kind, norms.data_ptr(),
                               codes.data_ptr(), status.data_ptr(), stream), "qsgd_bbit_encode_ef")
    return BbitEncoded(norms, codes, n, d, b, seed, status)


def bbit_decode(enc: BbitEncoded, out=None, status=None):
    torch = _torch()
    dev = enc.codes.device
    if out is None:
        out = torch.empty(enc.n, dtype=torch.float32, device=dev)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    _check(qsgd_bbit_decode(enc.norms.data_ptr(), enc.codes.data_ptr(), enc.n, enc.d, enc.b, out.data_ptr(),
                            status.data_ptr(), stream), "qsgd_bbit_decode")
    return out, status


def bbit_decode_accumulate(encs, out, status=None):
    torch = _torch()
    e0 = encs[0]
    dev = out.device
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    _check(qsgd_bbit_decode_accumulate([e.norms.data_ptr() for e in encs], [e.codes.data_ptr() for e in encs],
                                       len(encs), e0.n, e0.d, e0.b, out.data_ptr(), status.data_ptr(), stream),
           "qsgd_bbit_decode_accumulate")
    return out, status

"""Helpers of the GPU parity tests: run the CUDA path through the C ABI, compare
with the oracle.  The oracle never sees a value produced by the CUDA path except
the per-bucket norms, which the wire format lets any conforming encoder choose
within 1e-6 relative error; it then re-quantises with those norms."""

import numpy as np

NORM_RTOL = 1e-6


def torch_mod():
    import torch

    return torch


def binding():
    from quantized_gradient_compression_b200 import binding as B

    return B


def device_vector(v: np.ndarray, misalign: int = 0):
    """v on the GPU; misalign > 0 places it `misalign` floats past a 256-byte boundary."""
    torch = torch_mod()
    if misalign == 0:
        return torch.from_numpy(np.ascontiguousarray(v)).cuda()
    buf = torch.empty(v.size + misalign, dtype=torch.float32, device="cuda")
    x = buf[misalign:]
    x.copy_(torch.from_numpy(np.ascontiguousarray(v)))
    return x


def gpu_encode(x, d: int, s: int, seed: int):
    torch = torch_mod()
    B = binding()
    enc = B.encode(x, d, s, seed)
    torch.cuda.synchronize()
    offsets = enc.offsets.cpu().numpy().view(np.uint64)
    nwords = (int(offsets[-1]) + 31) // 32
    words = enc.words[:nwords].cpu().numpy().view(np.uint32).copy()
    return enc, words, offsets.copy(), int(enc.status.item())


def gpu_decode(enc):
    torch = torch_mod()
    B = binding()
    out, st = B.decode(enc)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(st.item())


def extract_bits(words: np.ndarray, begin: int, end: int) -> np.ndarray:
    """The bits [begin, end) of an MSB-first stream as a new zero-padded word array."""
    nbits = end - begin
    nw = (nbits + 31) // 32
    w64 = np.concatenate([words.astype(np.uint64), np.zeros(2, np.uint64)])
    idx = (begin >> 5) + np.arange(nw, dtype=np.int64)
    sh = np.uint64(begin & 31)
    hi = w64[idx]
    lo = w64[idx + 1]
    out = ((hi << sh) | (lo >> (np.uint64(32) - sh))) & np.uint64(0xFFFFFFFF) if sh else hi
    out = out.astype(np.uint32)
    if nbits % 32:
        out[-1] &= np.uint32((0xFFFFFFFF << (32 - nbits % 32)) & 0xFFFFFFFF)
    return out


def stream_norms(words: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    """The 32-bit norm field at the start of every bucket."""
    starts = offsets[:-1].astype(np.int64)
    w64 = np.concatenate([words.astype(np.uint64), np.zeros(2, np.uint64)])
    hi = w64[starts >> 5]
    lo = w64[(starts >> 5) + 1]
    sh = (starts & 31).astype(np.uint64)
    val = ((hi << sh) | (lo >> (np.uint64(32) - sh))) & np.uint64(0xFFFFFFFF)
    val = np.where(sh == 0, hi, val).astype(np.uint32)
    return val.view(np.float32)


def check_norms(gnorms: np.ndarray, onorms: np.ndarray):
    zero = onorms == 0
    assert np.array_equal(gnorms[zero].view(np.uint32), onorms[zero].view(np.uint32))
    rel = np.abs(gnorms[~zero].astype(np.float64) - onorms[~zero]) / onorms[~zero]
    assert rel.size == 0 or float(rel.max()) <= NORM_RTOL, float(rel.max())
    return float(rel.max()) if rel.size else 0.0


def check_parity(o, v: np.ndarray, d: int, s: int, seed: int, misalign: int = 0, decode=True):
    """Full-vector parity: norms within 1e-6, re-quantised stream and offsets
    bit-exact, decoded fp32 bit-exact, status equal."""
    x = device_vector(v, misalign)
    enc, words, offsets, status = gpu_encode(x, d, s, seed)
    nb = (v.size + d - 1) // d
    assert offsets.size == nb + 1
    own_words, own_offsets, own_norms, own_status = o.encode(v, d, s, seed)
    assert status == own_status
    gnorms = stream_norms(words, offsets) if nb else np.zeros(0, np.float32)
    check_norms(gnorms, own_norms)
    r_words, r_offsets, _, _ = o.encode(v, d, s, seed, norms_in=gnorms)
    assert np.array_equal(offsets, r_offsets)
    assert np.array_equal(words, r_words)
    if decode:
        out, st = gpu_decode(enc)
        ref, rst = o.decode(words, offsets, v.size, d, s)
        assert st == rst == 0
        assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))
    return enc, words, offsets

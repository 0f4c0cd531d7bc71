"""Malformed input through the C ABI: the decoders flag it, stay inside the
bucket, and finish.  All corruption is made on the host; nothing faults a GPU."""

import numpy as np
import pytest

from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu

PAD = 4096
SENTINEL = np.uint32(0x7FC0DEAD)  # a NaN pattern no decoder writes


def _encode(n, d, s, seed=3):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    v = W.normal(n, 21)
    x = torch.from_numpy(v).cuda()
    enc = B.encode(x, d, s, seed)
    torch.cuda.synchronize()
    offs = enc.offsets.cpu().numpy().view(np.uint64).copy()
    words = enc.words.cpu().numpy().view(np.uint32).copy()
    return enc, words, offs


def _decode_guarded(words, offs, n, d, s, accumulate=False):
    """Decodes host arrays on the GPU into the middle of a sentinel-filled buffer."""
    import torch
    from quantized_gradient_compression_b200 import binding as B

    w = torch.from_numpy(words.view(np.int32).copy()).cuda()
    o = torch.from_numpy(offs.view(np.int64).copy()).cuda()
    buf = torch.from_numpy(np.full(n + 2 * PAD, SENTINEL, dtype=np.uint32).view(np.int32)).cuda()
    out = buf[PAD:PAD + n].view(torch.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    if accumulate:
        out.zero_()
        rc = B.qsgd_decode_accumulate([w.data_ptr()], [w.numel()], [o.data_ptr()], 1, n, d, s,
                                      out.data_ptr(), st.data_ptr(), stream)
    else:
        rc = B.qsgd_decode(w.data_ptr(), w.numel(), o.data_ptr(), n, d, s, out.data_ptr(),
                           st.data_ptr(), stream)
    assert rc == 0
    torch.cuda.synchronize()
    host = buf.cpu().numpy().view(np.uint32)
    assert np.all(host[:PAD] == SENTINEL) and np.all(host[PAD + n:] == SENTINEL), "write outside the output"
    return host[PAD:PAD + n].view(np.float32), int(st.item())


@pytest.mark.parametrize("d", [512, 3, 8192])
@pytest.mark.parametrize("accumulate", [False, True])
@pytest.mark.parametrize("kind", ["truncate", "swap", "beyond_stream", "short_bucket", "nan_norm",
                                  "negative_norm", "level_above_s", "underflowing_scale"])
def test_flagged_corruption(kind, d, accumulate):
    n, s = 50_000, 8
    enc, words, offs = _encode(n, d, s)
    nb = offs.size - 1
    b = min(5, nb - 2)
    if kind == "truncate":
        offs[b + 1] -= 3
    elif kind == "swap":
        offs[b], offs[b + 1] = offs[b + 1], offs[b]
    elif kind == "beyond_stream":
        offs[nb] = np.uint64(words.size * 32 + 64)
    elif kind == "short_bucket":
        offs[b + 1] = offs[b] + np.uint64(16)
    elif kind in ("nan_norm", "negative_norm", "level_above_s", "underflowing_scale"):
        # rebuild bucket b as a hand-made bucket of exactly 32 + len bits
        start = int(offs[b])
        end = int(offs[b + 1])
        bits = "".join(format(int(x), "032b") for x in words)
        if kind == "nan_norm":
            body = "01111111110000000000000000000000"
        elif kind == "negative_norm":
            body = "10111111100000000000000000000000"  # -1.0f with records after it
        elif kind == "underflowing_scale":
            # norm 2^-149: norm / s rounds to zero; record gap 1, sign 1, k 1
            body = "0" * 31 + "1" + "0" + "1" + "0"
        else:
            # norm 1.0, record gap 1, sign 0, k = 9 > s = 8: omega(9) = 1110010
            body = "00111111100000000000000000000000" + "0" + "0" + "1110010"
        body = body + "0" * max(0, end - start - len(body))
        body = body[:end - start]
        bits = bits[:start] + body + bits[end:]
        words = np.array([int(bits[32 * i:32 * i + 32], 2) for i in range(words.size)], dtype=np.uint32)
    out, st = _decode_guarded(words, offs, n, d, s, accumulate)
    assert st & 2, "BAD_STREAM expected"


@pytest.mark.parametrize("d", [512, 3])
def test_random_bit_flips_terminate_in_bounds(d):
    rng = np.random.default_rng(0)
    n, s = 30_000, 16
    enc, words, offs = _encode(n, d, s)
    used = (int(offs[-1]) + 31) // 32
    for _ in range(5):
        w = words.copy()
        idx = rng.integers(0, used, size=20)
        w[idx] ^= np.uint32(1) << rng.integers(0, 32, size=20).astype(np.uint32)
        _decode_guarded(w, offs, n, d, s)  # status may or may not be set; bounds are checked


@pytest.mark.parametrize("d", [512, 132, 2048])
def test_corruption_stays_in_its_buckets(oracle_lib, d):
    """Bit flips inside some buckets leave every other bucket exactly as the oracle
    decodes the intact stream (the decoders read a bucket's bits only)."""
    rng = np.random.default_rng(d)
    n, s = 60_000, 16
    enc, words, offs = _encode(n, d, s)
    ref, _ = oracle_lib.decode(words, offs, n, d, s)
    nb = offs.size - 1
    hit = np.unique(rng.integers(0, nb, size=max(2, nb // 8)))
    w = words.copy()
    for b in hit:
        lo, hi = int(offs[b]) + 32, int(offs[b + 1])
        if hi <= lo:
            continue
        for pos in rng.integers(lo, hi, size=3):
            w[pos >> 5] ^= np.uint32(1) << np.uint32(31 - (pos & 31))
    out, st = _decode_guarded(w, offs, n, d, s)
    keep = np.ones(n, dtype=bool)
    for b in hit:
        keep[b * d:min(n, (b + 1) * d)] = False
    assert np.array_equal(out[keep].view(np.uint32), ref[keep].view(np.uint32))


def test_capacity_and_workspace_errors():
    import torch
    from quantized_gradient_compression_b200 import binding as B

    n, d, s = 10_000, 512, 16
    x = torch.zeros(n, dtype=torch.float32, device="cuda")
    cap = B.qsgd_max_encoded_words(n, d, s)
    words = torch.empty(cap, dtype=torch.int32, device="cuda")
    offs = torch.empty((n + d - 1) // d + 1, dtype=torch.int64, device="cuda")
    ws_bytes = B.qsgd_encode_workspace_bytes(n, d, s)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    h = torch.cuda.current_stream().cuda_stream
    assert B.qsgd_encode(x.data_ptr(), n, d, s, 0, words.data_ptr(), cap - 1, offs.data_ptr(), ws.data_ptr(),
                         ws_bytes, st.data_ptr(), h) == B.QSGD_ERR_CAPACITY
    assert B.qsgd_encode(x.data_ptr(), n, d, s, 0, words.data_ptr(), cap, offs.data_ptr(), ws.data_ptr(),
                         ws_bytes - 256, st.data_ptr(), h) == B.QSGD_ERR_WORKSPACE
    assert B.qsgd_encode(x.data_ptr(), n, d, s, 0, words.data_ptr(), cap, offs.data_ptr() + 4, ws.data_ptr(),
                         ws_bytes, st.data_ptr(), h) == B.QSGD_ERR_ARG
    assert B.qsgd_encode(x.data_ptr(), n, d, s, 0, words.data_ptr(), cap, offs.data_ptr(), ws.data_ptr(),
                         ws_bytes, st.data_ptr(), h) == B.QSGD_OK
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_nonfinite_input_status():
    import torch
    from quantized_gradient_compression_b200 import binding as B

    v = W.normal(4096, 2)
    v[100] = np.nan
    v[1500] = np.inf
    enc = B.encode(torch.from_numpy(v).cuda(), 512, 16, 0)
    torch.cuda.synchronize()
    assert int(enc.status.item()) & B.QSGD_ST_NONFINITE


@pytest.mark.parametrize("d,misalign", [(3, 0), (512, 1)])
def test_epoch_wrap_clears_stale_entries(oracle_lib, d, misalign):
    """The one-pass encoder tags workspace entries with a 24-bit call epoch.  Entries
    planted with epoch 0 and the "prefix ready" state would fool the call that runs
    with epoch 0.  The call that wraps the epoch (epoch 0xFFFFFF) must clear them, so
    that the next call, with epoch 0, still writes the oracle's stream.  (d = 3, and
    d = 512 on misaligned input, take the one-pass encoder.)"""
    import torch
    from gpu_common import check_norms, device_vector, stream_norms
    from quantized_gradient_compression_b200 import binding as B

    s, seed = 16, 9
    ws = torch.zeros(4 << 20, dtype=torch.uint8, device="cuda")
    ws[256:].view(torch.int64).fill_((2 << 38) | 12345)  # epoch 0, prefix ready, a wrong value
    ws[8:12].view(torch.int32).fill_(0xFFFFFF)  # the control block's epoch
    h = torch.cuda.current_stream().cuda_stream
    # the wrapping call has one tile; the next call's look-back reads entries past it
    for call, n in enumerate((4_000, 40_000)):
        v = W.layered(n, 4)
        x = device_vector(v, misalign)
        nb = (n + d - 1) // d
        cap = B.qsgd_max_encoded_words(n, d, s)
        assert ws.numel() >= B.qsgd_encode_workspace_bytes(n, d, s)
        words = torch.zeros(cap, dtype=torch.int32, device="cuda")
        offs = torch.zeros(nb + 1, dtype=torch.int64, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert B.qsgd_encode(x.data_ptr(), n, d, s, seed, words.data_ptr(), cap, offs.data_ptr(), ws.data_ptr(),
                             ws.numel(), st.data_ptr(), h) == B.QSGD_OK
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert int(ws[8:12].view(torch.int32).item()) == call  # 0xFFFFFF + 1 wraps to 0, then 1
        o = offs.cpu().numpy().view(np.uint64)
        w = words[:(int(o[-1]) + 31) // 32].cpu().numpy().view(np.uint32)
        gn = stream_norms(w, o)
        _, _, onorms, _ = oracle_lib.encode(v, d, s, seed)
        check_norms(gn, onorms)
        r_words, r_offsets, _, _ = oracle_lib.encode(v, d, s, seed, norms_in=gn)
        assert np.array_equal(o, r_offsets) and np.array_equal(w, r_words)

"""Data-parallel exchange of QSGD encodings: one process per GPU, torch.distributed.

The definition paragraph of "QSGD (Quantized Stochastic Gradient Descent) with Elias
Coding" (AIMech curated entry) sets the codec in distributed data-parallel
optimisation.  Each node quantises and encodes its gradient, the nodes exchange the
encodings, and each node applies the mean of the K decoded gradients.  One step here:

1. Encode this rank's gradient with the library, optionally through the
   error-feedback memory.
2. All-gather each rank's stream length (one int64 per rank).
3. All-gather the offsets headers, (nb + 1) int64 per rank.
4. All-gather the streams, each padded to the longest.  A host read of the gathered
   lengths sizes this gather: it is the step's one synchronisation.
5. Decode the mean of the K streams with the library.

The b-bit codec needs no lengths: its norms and codes have fixed sizes.

torch.distributed carries only bytes: NCCL over NVLink / NVSwitch on B200, gloo on the
CPU in tests.  Every arithmetic step runs in the CUDA library, reached through a codec
object.  The default codec is the library's; it takes CUDA tensors only, so there is
no CPU path.  Every rank takes the same collective steps in the same order.  Rank r
encodes with seed + r, so the ranks' random words are independent.
"""

from __future__ import annotations

from dataclasses import dataclass

from . import binding as B


def _torch():
    import torch

    return torch


def rank_seed(seed: int, rank: int) -> int:
    """The Philox seed rank `rank` encodes with at step seed `seed`."""
    return (seed + rank) & 0xFFFFFFFFFFFFFFFF


# ---------------------------------------------------------------------------
# Codecs: the arithmetic of a step, behind four calls
# ---------------------------------------------------------------------------
class LibraryCodec:
    """The CUDA library: Elias-omega streams on the device."""

    def __init__(self, n: int, d: int, s: int, device, norm_kind: int = B.QSGD_NORM_L2):
        torch = _torch()
        self.n, self.d, self.s, self.norm_kind = n, d, s, norm_kind
        self.device = torch.device(device)
        self.nb = B.qsgd_num_buckets(n, d)
        self.cap = B.qsgd_max_encoded_words(n, d, s)
        self.words = torch.empty(max(self.cap, 1), dtype=torch.int32, device=self.device)
        self.offsets = torch.empty(self.nb + 1, dtype=torch.int64, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)

    def encode(self, grad, memory, seed: int):
        """Encodes grad (through memory when given); returns (words, offsets)."""
        if memory is None:
            B.encode(grad, self.d, self.s, seed, words=self.words, offsets=self.offsets, status=self.status,
                     norm_kind=self.norm_kind)
        else:
            B.encode_ef(grad, memory, self.d, self.s, seed, words=self.words, offsets=self.offsets,
                        status=self.status, norm_kind=self.norm_kind)
        return self.words, self.offsets

    def stream_bits(self, offsets):
        """This rank's stream length in bits, as a one-element int64 tensor (no host read)."""
        return offsets[self.nb:self.nb + 1]

    def decode_mean(self, words, num_words: int, offsets, K: int, out):
        """out = mean of the K streams laid out as rank-major slices of words / offsets."""
        torch = _torch()
        stream = torch.cuda.current_stream(out.device).cuda_stream
        w0, o0 = words.data_ptr(), offsets.data_ptr()
        rc = B.qsgd_decode_mean([w0 + 4 * num_words * j for j in range(K)], [num_words] * K,
                                [o0 + 8 * (self.nb + 1) * j for j in range(K)], K, self.n, self.d, self.s,
                                out.data_ptr(), self.status.data_ptr(), stream)
        if rc != B.QSGD_OK:
            raise RuntimeError("qsgd_decode_mean: %s" % B.qsgd_error_string(rc))
        return out


class LibraryBbitCodec:
    """The CUDA library: fixed-width b-bit codes on the device."""

    def __init__(self, n: int, d: int, b: int, device, norm_kind: int = B.QSGD_NORM_L2):
        torch = _torch()
        self.n, self.d, self.b, self.norm_kind = n, d, b, norm_kind
        self.device = torch.device(device)
        self.nb = B.qsgd_num_buckets(n, d)
        self.cw = B.qsgd_bbit_code_words(n, b)
        self.norms = torch.empty(max(self.nb, 1), dtype=torch.float32, device=self.device)
        self.codes = torch.empty(max(self.cw, 1), dtype=torch.int32, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)

    def encode(self, grad, memory, seed: int):
        if memory is None:
            B.bbit_encode(grad, self.d, self.b, seed, norms=self.norms, codes=self.codes, status=self.status,
                          norm_kind=self.norm_kind)
        else:
            B.bbit_encode_ef(grad, memory, self.d, self.b, seed, norms=self.norms, codes=self.codes,
                             status=self.status, norm_kind=self.norm_kind)
        return self.norms, self.codes

    def decode_mean(self, norms, codes, K: int, out):
        torch = _torch()
        stream = torch.cuda.current_stream(out.device).cuda_stream
        n0, c0 = norms.data_ptr(), codes.data_ptr()
        m_n, m_c = self.norms.numel(), self.codes.numel()
        rc = B.qsgd_bbit_decode_mean([n0 + 4 * m_n * j for j in range(K)], [c0 + 4 * m_c * j for j in range(K)],
                                     K, self.n, self.d, self.b, out.data_ptr(), self.status.data_ptr(), stream)
        if rc != B.QSGD_OK:
            raise RuntimeError("qsgd_bbit_decode_mean: %s" % B.qsgd_error_string(rc))
        return out


# ---------------------------------------------------------------------------
# The exchange
# ---------------------------------------------------------------------------
def _all_gather(out, inp, group):
    """out = the ranks' inp, rank-major (a copy in a process without a group)."""
    import torch.distributed as dist

    if dist.is_initialized():
        dist.all_gather_into_tensor(out, inp, group=group)
    else:
        out.copy_(inp)


@dataclass
class StepInfo:
    """What one exchange step moved (bytes this rank sent into the gathers)."""

    max_words: int
    sent_bytes: int


class EliasExchange:
    """All-gather exchange of Elias-omega streams and the mean of the K decodes."""

    def __init__(self, codec, group=None):
        import torch.distributed as dist

        self.codec = codec
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.last = StepInfo(0, 0)

    def _gather(self, out, inp):
        _all_gather(out, inp, self.group)

    def step(self, grad, seed: int, memory=None, out=None):
        """Exchanges this rank's encoding of grad; returns the mean of all ranks' decodes."""
        torch = _torch()
        K = self.world
        words, offsets = self.codec.encode(grad, memory, rank_seed(seed, self.rank))
        # stream lengths, then the padded payload
        bits = self.codec.stream_bits(offsets)
        all_bits = torch.empty(K, dtype=torch.int64, device=bits.device)
        self._gather(all_bits, bits)
        max_words = max(1, (int(all_bits.max().item()) + 31) // 32)
        g_off = torch.empty(K * offsets.numel(), dtype=torch.int64, device=offsets.device)
        self._gather(g_off, offsets)
        g_words = torch.empty(K * max_words, dtype=torch.int32, device=words.device)
        self._gather(g_words, words[:max_words])
        if out is None:
            out = torch.empty(grad.numel(), dtype=torch.float32, device=grad.device)
        self.codec.decode_mean(g_words, max_words, g_off, K, out)
        self.last = StepInfo(max_words, 8 + 8 * offsets.numel() + 4 * max_words)
        return out


class BbitExchange:
    """All-gather exchange of b-bit norms and codes (fixed sizes) and the mean."""

    def __init__(self, codec, group=None):
        import torch.distributed as dist

        self.codec = codec
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0

    def _gather(self, out, inp):
        _all_gather(out, inp, self.group)

    def step(self, grad, seed: int, memory=None, out=None):
        torch = _torch()
        K = self.world
        norms, codes = self.codec.encode(grad, memory, rank_seed(seed, self.rank))
        g_norms = torch.empty(K * norms.numel(), dtype=norms.dtype, device=norms.device)
        self._gather(g_norms, norms)
        g_codes = torch.empty(K * codes.numel(), dtype=codes.dtype, device=codes.device)
        self._gather(g_codes, codes)
        if out is None:
            out = torch.empty(grad.numel(), dtype=torch.float32, device=grad.device)
        return self.codec.decode_mean(g_norms, g_codes, K, out)

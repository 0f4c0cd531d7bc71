"""qsgd_encode_static_ws: the encoder for callers that cannot allocate device memory.

Some callers may not call cudaMalloc where they compress a gradient (inside a
caching allocator's callbacks, in a communication progress thread that must not
take the allocator lock, or in an embedding that only hands over input and output
buffers).  This entry point keeps the encoder's scan state in a fixed device array
of the library instead of a caller workspace.  Its stream must be bit-identical to
the one qsgd_encode writes.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test.  It passes on its own in a fresh process
(the array starts zeroed) and after the other tests.
"""

import numpy as np
import pytest

from quantized_gradient_compression_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _static_encode(x, n, d, s, seed):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    cap = B.qsgd_max_encoded_words(n, d, s)
    words = torch.empty(cap, dtype=torch.int32, device="cuda")
    offsets = torch.empty((n + d - 1) // d + 1, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = B.qsgd_encode_static_ws(x.data_ptr(), n, d, s, seed, words.data_ptr(), cap, offsets.data_ptr(),
                                 status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == B.QSGD_OK, B.qsgd_error_string(rc)
    return words, offsets, status


def _compare(v, d, s, seed):
    import torch
    from quantized_gradient_compression_b200 import binding as B

    n = v.size
    x = torch.from_numpy(v).cuda()
    ref = B.encode(x, d, s, seed)                       # caller-workspace entry point
    words, offsets, status = _static_encode(x, n, d, s, seed)
    torch.cuda.synchronize()
    ro = ref.offsets.cpu().numpy().view(np.uint64)
    so = offsets.cpu().numpy().view(np.uint64)
    assert np.array_equal(ro, so)
    used = (int(ro[-1]) + 31) // 32
    assert np.array_equal(ref.words[:used].cpu().numpy(), words[:used].cpu().numpy())
    assert int(ref.status.item()) == int(status.item()) == 0


def test_static_workspace_matches_encode_on_consecutive_calls():
    # two calls in a row of different shapes (fast path, then the general path),
    # then the first shape again on the state the second call left behind
    _compare(W.layered(300_001, 7), 512, 16, 5)
    _compare(W.normal(100_003, 8), 3, 4, 6)
    _compare(W.layered(300_001, 7), 512, 16, 5)


def test_static_workspace_rejects_problems_above_its_limit():
    from quantized_gradient_compression_b200 import binding as B

    limit = B.qsgd_static_workspace_limit()
    assert limit == 4 << 20
    n, d, s = 1 << 30, 512, 16
    assert B.qsgd_encode_workspace_bytes(n, d, s) > limit
    # rejected on the host before any pointer is used
    assert B.qsgd_encode_static_ws(0, n, d, s, 0, 0, 0, 0, 0, 0) == B.QSGD_ERR_STATIC_LIMIT

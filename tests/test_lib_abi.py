"""The C-ABI library loads on the CPU and exports every entry point of include/qsgd.h.

No compute call is made here: only host-side size queries and argument checks
that return before any CUDA call.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "qsgd.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^QSGD_API\s+[\w\s\*]+?\b(qsgd_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from quantized_gradient_compression_b200 import build

    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = declared_symbols()
    for want in ["qsgd_encode", "qsgd_decode", "qsgd_decode_accumulate", "qsgd_max_encoded_words",
                 "qsgd_encode_workspace_bytes", "qsgd_num_buckets", "qsgd_error_string",
                 "qsgd_bbit_encode", "qsgd_bbit_decode", "qsgd_bbit_decode_accumulate", "qsgd_bbit_code_words"]:
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_binding_exposes_same_names():
    from quantized_gradient_compression_b200 import binding

    for name in declared_symbols():
        assert hasattr(binding, name), name
        assert name in binding.EXPORTED


def test_size_queries_match_oracle_bound(oracle_lib):
    from quantized_gradient_compression_b200 import binding as B

    for n, d, s in [(1, 1, 1), (7, 3, 2), (25_557_032, 512, 16), (60_192_808, 8192, 1),
                    (65_536, 65_536, 256), (1 << 30, 512, 256), (1000, 7, 1 << 22)]:
        assert B.qsgd_num_buckets(n, d) == (n + d - 1) // d
        if n <= 100_000:
            assert B.qsgd_max_encoded_words(n, d, s) == oracle_lib.capacity_words(n, d, s)
        else:
            nb = (n + d - 1) // d
            bits = 32 * nb + n * (2 + oracle_lib.omega_len(s))
            assert B.qsgd_max_encoded_words(n, d, s) == (bits + 31) // 32
        assert B.qsgd_encode_workspace_bytes(n, d, s) >= 256


def test_invalid_parameters_are_rejected_on_the_host():
    from quantized_gradient_compression_b200 import binding as B

    assert B.qsgd_max_encoded_words(10, 0, 4) == 0
    assert B.qsgd_max_encoded_words(10, 4, 0) == 0
    assert B.qsgd_max_encoded_words(10, 4, (1 << 22) + 1) == 0
    # argument errors are detected before any CUDA call
    assert B.qsgd_encode(0, 10, 0, 4, 0, 0, 0, 8, 0, 0, 8, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_encode(256, 10, 4, 4, 0, 256, 100, 256, 256, 1 << 20, 0, 0) == B.QSGD_ERR_ARG  # no status
    assert B.qsgd_encode(256, 100, 4, 4, 0, 256, 1, 256, 256, 1 << 20, 256, 0) == B.QSGD_ERR_CAPACITY
    assert B.qsgd_encode(256, 100, 4, 4, 0, 256, 1000, 256, 256, 1, 256, 0) == B.QSGD_ERR_WORKSPACE
    assert B.qsgd_encode(256, 100, 4, 4, 0, 256, 1000, 257, 256, 1 << 20, 256, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_decode(256, 10, 256, 10, 4, 0, 256, 256, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_decode_accumulate([], [], [], 0, 10, 4, 4, 256, 256, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_error_string(B.QSGD_ERR_CAPACITY).startswith("output capacity")
    assert "sm_100a" in B.qsgd_version()


def test_library_is_sm100a_only():
    from quantized_gradient_compression_b200 import build

    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "-fmad=false" in flags
    assert "use_fast_math" not in flags


def test_bbit_size_query_and_argument_checks(oracle_lib):
    from quantized_gradient_compression_b200 import binding as B

    for n in (0, 1, 15, 16, 17, 25_557_032):
        for b in (2, 4, 8):
            assert B.qsgd_bbit_code_words(n, b) == oracle_lib.bbit_code_words(n, b)
    # widths other than 2, 4, 8 and null pointers are refused before any CUDA call
    assert B.qsgd_bbit_encode(256, 10, 4, 3, 0, 256, 256, 256, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_encode(0, 10, 4, 4, 0, 256, 256, 256, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_decode(256, 256, 10, 4, 16, 256, 256, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_decode_accumulate([], [], 0, 10, 4, 4, 256, 256, 0) == B.QSGD_ERR_ARG


def test_norm_kind_checked():
    from quantized_gradient_compression_b200 import binding as B

    assert B.QSGD_NORM_L2 == 0 and B.QSGD_NORM_MAX == 1
    # an unknown norm kind is refused before any CUDA call
    assert B.qsgd_encode_ex(256, 10, 4, 4, 0, 2, 256, 100, 256, 256, 4096, 256, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_encode_ex(256, 10, 4, 4, 0, 7, 256, 256, 256, 0) == B.QSGD_ERR_ARG


def test_error_feedback_arguments_checked():
    from quantized_gradient_compression_b200 import binding as B

    A = 1 << 20  # fake device addresses: every call below is refused before a CUDA call
    # g and e overlap
    assert B.qsgd_encode_ef(A, A + 64, 100, 4, 4, 0, 0, A * 8, 10_000, A * 16, A * 32, 1 << 20, A * 64, 0) \
        == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_encode_ef(A, A + 64, 100, 4, 4, 0, 0, A * 8, A * 16, A * 64, 0) == B.QSGD_ERR_ARG
    # a null memory, a misaligned gradient, an unknown norm kind
    assert B.qsgd_encode_ef(A, 0, 100, 4, 4, 0, 0, A * 8, 10_000, A * 16, A * 32, 1 << 20, A * 64, 0) \
        == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_encode_ef(A + 2, A * 4, 100, 4, 4, 0, 0, A * 8, A * 16, A * 64, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_encode_ef(A, A * 4, 100, 4, 4, 0, 5, A * 8, A * 16, A * 64, 0) == B.QSGD_ERR_ARG


def test_mean_arguments_checked():
    from quantized_gradient_compression_b200 import binding as B

    A = 1 << 20
    # K out of range, a null stream among valid ones, a misaligned offsets array:
    # refused before any launch
    assert B.qsgd_decode_mean([], [], [], 0, 100, 4, 4, A, A, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_decode_mean([A, 0], [10, 10], [A * 2, A * 2], 2, 100, 4, 4, A * 4, A * 8, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_decode_mean([A, A], [10, 10], [A * 2, A * 2 + 4], 2, 100, 4, 4, A * 4, A * 8, 0) \
        == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_decode_mean([A, 0], [A, A], 2, 100, 4, 4, A * 4, A * 8, 0) == B.QSGD_ERR_ARG
    assert B.qsgd_bbit_decode_mean([A], [A], 1, 100, 4, 3, A * 4, A * 8, 0) == B.QSGD_ERR_ARG


def test_product_path_fails_loudly_without_the_library(tmp_path):
    """No CPU fallback: the binding refuses to import when the CUDA library is absent."""
    import importlib.util
    import shutil

    src = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "quantized_gradient_compression_b200", "binding.py")
    shutil.copy(src, tmp_path / "binding.py")  # a package directory with no .so in it
    spec = importlib.util.spec_from_file_location("binding_without_lib", tmp_path / "binding.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="not built"):
        spec.loader.exec_module(mod)


def test_library_codec_takes_cuda_tensors_only():
    import torch
    from quantized_gradient_compression_b200 import binding as B

    with pytest.raises(AssertionError):
        B.encode(torch.zeros(1024), 512, 16, 0)

"""B200-native QSGD gradient codec.

The codec (bucket L2 norm, unbiased stochastic rounding to s+1 levels, Elias-omega
coding of the sparse result, the matching decoder and a decode-and-sum of K
streams) runs in hand-written CUDA for sm_100a behind a C ABI
(``include/qsgd.h``).  ``binding`` is a thin ctypes layer over that library with
the same entry-point names; it raises at import if the library is missing.

``workloads`` (seeded synthetic gradients) imports without the CUDA library.
"""

_BINDING_NAMES = {
    "qsgd_num_buckets", "qsgd_max_encoded_words", "qsgd_encode_workspace_bytes",
    "qsgd_encode", "qsgd_decode", "qsgd_decode_accumulate", "qsgd_error_string",
    "qsgd_version", "QsgdError", "Encoded", "encode", "decode", "decode_accumulate",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding

        return getattr(binding, name)
    raise AttributeError(name)

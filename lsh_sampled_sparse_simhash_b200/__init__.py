"""B200 (sm_100a) LSH-sampled decode attention (MagicPIG hot path).

The compute lives in ``libmagicpig_b200.so`` (hand-written CUDA kernels behind
the C ABI of ``include/magicpig.h``); this package is a thin ctypes binding
that marshals torch tensors (device memory and streams only) into those calls.
There is no fallback: if the library is missing or cannot load, every call
raises.
"""
from ._binding import (  # noqa: F401
    MagicPIGError,
    Shape,
    append_token,
    append_token_q8,
    auto_planes,
    codes_bytes,
    codes_shape,
    decode_attend,
    decode_attend_noalloc,
    decode_attend_q8,
    decode_workspace_bytes,
    hash_keys,
    hash_keys_range,
    hash_queries,
    library,
    library_path,
    quantize_keys,
    read_status,
    status_string,
    MP_OK,
    MP_ERR_ARG,
    MP_ERR_SHAPE,
    MP_ERR_ALIGN,
    MP_ERR_CAPACITY,
    MP_ERR_WORKSPACE,
    MP_ERR_CUDA,
    MP_ERR_TOO_LARGE,
    MP_CODES_AUTO,
    MP_CODES_BYTES,
    MP_CODES_PLANES,
    MP_CODES_AUTO_PLANES_MIN,
    Q8_ROW_BYTES,
    MP_PATH_AUTO,
    MP_PATH_SPLIT,
    MP_PATH_FUSED,
    MP_PATH_TC,
)

__all__ = [
    "MagicPIGError", "Shape", "append_token", "append_token_q8", "auto_planes", "codes_bytes", "codes_shape", "decode_attend",
    "decode_attend_noalloc", "decode_attend_q8", "quantize_keys",
    "decode_workspace_bytes", "hash_keys", "hash_keys_range", "hash_queries", "library", "library_path", "read_status",
    "status_string",
]

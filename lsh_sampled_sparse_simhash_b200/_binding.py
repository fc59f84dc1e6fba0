"""ctypes binding of include/magicpig.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libmagicpig_b200.so")

MP_OK = 0
MP_ERR_ARG = -1
MP_ERR_SHAPE = -2
MP_ERR_ALIGN = -3
MP_ERR_CAPACITY = -4
MP_ERR_WORKSPACE = -5
MP_ERR_CUDA = -6
MP_ERR_TOO_LARGE = -7
MP_CODES_AUTO = 0
MP_CODES_BYTES = 1
MP_CODES_PLANES = 2
MP_PATH_AUTO = 0
MP_PATH_SPLIT = 1
MP_PATH_FUSED = 2
MP_PATH_TC = 3


class MagicPIGError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


class _CShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("batch", "n_q_heads", "n_kv_heads", "head_dim", "capacity", "k_bits", "n_tables",
                 "sink", "window", "code_layout")]


class _CDebug(ctypes.Structure):
    _fields_ = [("qcodes_in", ctypes.c_void_p), ("qcodes_out", ctypes.c_void_p),
                ("member_out", ctypes.c_void_p), ("path", ctypes.c_int32), ("skip_scan", ctypes.c_int32)]


MP_CODES_AUTO_PLANES_MIN = 1 << 21  # include/magicpig.h


def auto_planes(batch: int, n_kv_heads: int, capacity: int, k_bits: int) -> bool:
    """MP_CODES_AUTO: bit planes, except byte codes for K = 8 problems with
    fewer than MP_CODES_AUTO_PLANES_MIN (token, kv head) slots."""
    return k_bits != 8 or batch * n_kv_heads * capacity >= MP_CODES_AUTO_PLANES_MIN


@dataclasses.dataclass(frozen=True)
class Shape:
    """Problem shape (see mp_shape in include/magicpig.h)."""
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    capacity: int
    k_bits: int
    n_tables: int
    sink: int
    window: int
    code_layout: int = 0  # MP_CODES_AUTO

    @property
    def planes(self) -> bool:
        """Whether the key codes are bit planes (the library's rule for MP_CODES_AUTO)."""
        if self.code_layout == MP_CODES_AUTO:
            return auto_planes(self.batch, self.n_kv_heads, self.capacity, self.k_bits)
        return self.code_layout == MP_CODES_PLANES

    def c(self) -> _CShape:
        return _CShape(*dataclasses.astuple(self))


_lib = None


def library() -> ctypes.CDLL:
    """Loads the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise MagicPIGError(MP_ERR_CUDA, f"{library_path} not built (run __graft_entry__.build())")
        lib = ctypes.CDLL(library_path)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        SP = ctypes.POINTER(_CShape)
        lib.mp_codes_bytes.argtypes = [SP, ctypes.POINTER(SZ)]
        lib.mp_hash_keys.argtypes = [SP, P, P, P, I32, P, P, P]
        lib.mp_hash_keys_range.argtypes = [SP, P, P, I32, I32, P, P, P]
        lib.mp_hash_queries.argtypes = [SP, P, P, P, P]
        lib.mp_append_token.argtypes = [SP, P, P, P, P, P, P, P, P, P]
        lib.mp_decode_workspace_bytes.argtypes = [SP, I32, ctypes.POINTER(SZ)]
        lib.mp_decode_attend.argtypes = [SP, P, P, P, P, P, P, I32, P, P, P, P, SZ,
                                         ctypes.POINTER(_CDebug), P]
        lib.mp_decode_attend_noalloc.argtypes = [SP, P, P, P, P, P, P, I32, P, P, P, P, P]
        lib.mp_quantize_keys.argtypes = [SP, P, P, I32, I32, P, P]
        lib.mp_append_token_q8.argtypes = [SP, P, P, P, P, P, P, P, P, P, P]
        lib.mp_decode_attend_q8.argtypes = [SP, P, P, P, P, P, P, I32, P, P, P, P, SZ,
                                            ctypes.POINTER(_CDebug), P]
        lib.mp_read_status.argtypes = [P, ctypes.POINTER(I32), P]
        lib.mp_status_string.argtypes = [ctypes.c_int]
        lib.mp_status_string.restype = ctypes.c_char_p
        for f in ("mp_codes_bytes", "mp_hash_keys", "mp_hash_keys_range", "mp_hash_queries", "mp_append_token",
                  "mp_decode_workspace_bytes", "mp_decode_attend", "mp_decode_attend_noalloc",
                  "mp_quantize_keys", "mp_append_token_q8", "mp_decode_attend_q8", "mp_read_status"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def status_string(code: int) -> str:
    try:
        return library().mp_status_string(int(code)).decode()
    except MagicPIGError:
        return f"status {code}"


def _check(code: int, where: str):
    if code != MP_OK:
        raise MagicPIGError(code, where)


def _ptr(t) -> Optional[int]:
    """Device pointer of a torch tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def codes_bytes(shape: Shape) -> int:
    n = ctypes.c_size_t()
    _check(library().mp_codes_bytes(ctypes.byref(shape.c()), ctypes.byref(n)), "mp_codes_bytes")
    return n.value


def codes_shape(shape: Shape):
    """(dtype name, tensor shape) of the key codes: uint8 [B,Hkv,L,Ncap] for
    byte codes, int32 bit planes [B,Hkv,L,Ncap/32,K] for plane codes."""
    B, Hkv, L, K, N = shape.batch, shape.n_kv_heads, shape.n_tables, shape.k_bits, shape.capacity
    if not shape.planes:
        return "uint8", (B, Hkv, L, N)
    return "int32", (B, Hkv, L, N // 32, K)


def decode_workspace_bytes(shape: Shape, max_len: int) -> int:
    n = ctypes.c_size_t()
    _check(library().mp_decode_workspace_bytes(ctypes.byref(shape.c()), int(max_len), ctypes.byref(n)),
           "mp_decode_workspace_bytes")
    return n.value


def hash_keys(shape: Shape, keys, W, n_tokens: int, codes, seq_lens=None, status=None, stream=None):
    _check(library().mp_hash_keys(ctypes.byref(shape.c()), _ptr(keys), _ptr(W), _ptr(seq_lens), int(n_tokens),
                                  _ptr(codes), _ptr(status), _stream(stream)), "mp_hash_keys")


def hash_keys_range(shape: Shape, keys, W, first_token: int, n_tokens: int, codes, status=None, stream=None):
    """Hashes tokens [first_token, first_token + n_tokens) of every unit (a
    streamed prefill block; first_token a multiple of 128)."""
    _check(library().mp_hash_keys_range(ctypes.byref(shape.c()), _ptr(keys), _ptr(W), int(first_token),
                                        int(n_tokens), _ptr(codes), _ptr(status), _stream(stream)),
           "mp_hash_keys_range")


def hash_queries(shape: Shape, q, W, qcodes, stream=None):
    _check(library().mp_hash_queries(ctypes.byref(shape.c()), _ptr(q), _ptr(W), _ptr(qcodes), _stream(stream)),
           "mp_hash_queries")


def append_token(shape: Shape, k_new, v_new, W, k_cache, v_cache, codes, seq_lens, status=None, stream=None):
    _check(library().mp_append_token(ctypes.byref(shape.c()), _ptr(k_new), _ptr(v_new), _ptr(W),
                                     _ptr(k_cache), _ptr(v_cache), _ptr(codes), _ptr(seq_lens), _ptr(status),
                                     _stream(stream)), "mp_append_token")


def decode_attend(shape: Shape, q, W, codes, k_cache, v_cache, seq_lens, max_len: int, out, lse, n_sampled,
                  workspace, qcodes_in=None, qcodes_out=None, member_out=None, path: int = 0, skip_scan: bool = False,
                  stream=None):
    dbg = None
    if qcodes_in is not None or qcodes_out is not None or member_out is not None or path or skip_scan:
        dbg = ctypes.byref(_CDebug(_ptr(qcodes_in), _ptr(qcodes_out), _ptr(member_out), int(path),
                                   int(bool(skip_scan))))
    nbytes = workspace.numel() * workspace.element_size()
    _check(library().mp_decode_attend(ctypes.byref(shape.c()), _ptr(q), _ptr(W), _ptr(codes), _ptr(k_cache),
                                      _ptr(v_cache), _ptr(seq_lens), int(max_len), _ptr(out), _ptr(lse),
                                      _ptr(n_sampled), _ptr(workspace), nbytes, dbg, _stream(stream)),
           "mp_decode_attend")


def decode_attend_noalloc(shape: Shape, q, W, codes, k_cache, v_cache, seq_lens, max_len: int, out, lse,
                          n_sampled, status=None, stream=None):
    """mp_decode_attend with the library's fixed scratch array instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    _check(library().mp_decode_attend_noalloc(ctypes.byref(shape.c()), _ptr(q), _ptr(W), _ptr(codes),
                                              _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), int(max_len),
                                              _ptr(out), _ptr(lse), _ptr(n_sampled), _ptr(status),
                                              _stream(stream)), "mp_decode_attend_noalloc")


Q8_ROW_BYTES = 144  # MP_Q8_ROW_BYTES


def quantize_keys(shape: Shape, k_cache, k8, first_token: int = 0, n_tokens: Optional[int] = None,
                  seq_lens=None, stream=None):
    """Writes the int8 rows of key rows [first_token, first_token + n_tokens)
    (default: the whole capacity) into k8, int8 [B,Hkv,Ncap,144]: 128 int8
    values, then the fp32 record {power-of-two scale, squared norm of the
    int8 row times the scale, 0, 0}."""
    n = shape.capacity - int(first_token) if n_tokens is None else int(n_tokens)
    _check(library().mp_quantize_keys(ctypes.byref(shape.c()), _ptr(k_cache), _ptr(seq_lens), int(first_token), n,
                                      _ptr(k8), _stream(stream)), "mp_quantize_keys")


def append_token_q8(shape: Shape, k_new, v_new, W, k_cache, v_cache, codes, seq_lens, k8, status=None,
                    stream=None):
    _check(library().mp_append_token_q8(ctypes.byref(shape.c()), _ptr(k_new), _ptr(v_new), _ptr(W),
                                        _ptr(k_cache), _ptr(v_cache), _ptr(codes), _ptr(seq_lens), _ptr(k8),
                                        _ptr(status), _stream(stream)), "mp_append_token_q8")


def decode_attend_q8(shape: Shape, q, W, codes, k8, v_cache, seq_lens, max_len: int, out, lse, n_sampled,
                     workspace, qcodes_in=None, qcodes_out=None, member_out=None, path: int = 0, stream=None):
    """decode_attend with the K rows gathered from the int8 copy."""
    dbg = None
    if qcodes_in is not None or qcodes_out is not None or member_out is not None or path:
        dbg = ctypes.byref(_CDebug(_ptr(qcodes_in), _ptr(qcodes_out), _ptr(member_out), int(path)))
    nbytes = workspace.numel() * workspace.element_size()
    _check(library().mp_decode_attend_q8(ctypes.byref(shape.c()), _ptr(q), _ptr(W), _ptr(codes), _ptr(k8),
                                         _ptr(v_cache), _ptr(seq_lens), int(max_len), _ptr(out),
                                         _ptr(lse), _ptr(n_sampled), _ptr(workspace), nbytes, dbg,
                                         _stream(stream)), "mp_decode_attend_q8")


def read_status(workspace, stream=None) -> int:
    v = ctypes.c_int32()
    _check(library().mp_read_status(_ptr(workspace), ctypes.byref(v), _stream(stream)), "mp_read_status")
    return v.value

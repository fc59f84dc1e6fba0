"""Reference for the int8 key format of the reduced-precision attention gather.

TEST INFRASTRUCTURE ONLY (like the rest of this package).

The method reads the cached keys in their own precision; the int8 copy is an
opt-in variant of the library, so there is no passage of the method to cite
here.  The format is defined by the library's public header: one row k of d
bf16 values becomes

    s = 2^e, the smallest power of two with 127 s >= max_j |k_j|   (s = 0 for k = 0)
    q_j = round-half-to-even(k_j / s)                             (int8, |q_j| <= 127)
    meta = {s, |s q|^2, 0, 0}                                     (fp32 x 4 per row)

stored as one 144-byte row: the 128 int8 values, then the record.

and the attention then runs on k~ = s q.  This module writes that definition
out in fp64 numpy, one row at a time, so that a reader can check it by eye.
"""
from __future__ import annotations

import math

import numpy as np


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def row_scale(amax: float) -> float:
    """Smallest power of two s with 127 s >= amax (0 for amax = 0)."""
    if amax == 0.0:
        return 0.0
    e = math.frexp(amax)[1] - 8  # 127 * 2^(E - 8) < 2^(E - 1) <= amax: too small, so search upwards
    while 127.0 * math.ldexp(1.0, e) < amax:
        e += 1
    return math.ldexp(1.0, e)


def quantize_rows(k_bits: np.ndarray):
    """k_bits (bf16 bits) [..., d] -> (q int8 [..., d], s float32 [...])."""
    k = _bf16_to_f64(k_bits)
    flat = k.reshape(-1, k.shape[-1])
    q = np.zeros(flat.shape, np.int8)
    s = np.zeros(flat.shape[0], np.float32)
    for i, row in enumerate(flat):
        si = row_scale(float(np.max(np.abs(row))))
        if si > 0.0:
            # row / si is exact (si is a power of two); np.rint rounds half to even
            qi = np.rint(row / si)
            assert np.all(np.abs(qi) <= 127)
            q[i] = qi.astype(np.int8)
        s[i] = si
    return q.reshape(k.shape), s.reshape(k.shape[:-1])


def row_meta(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """The 16-byte record of each row, fp32 [..., 4] = {s, |s q|^2, 0, 0}.
    The squared norm is computed in fp64 and must be exact in fp32."""
    n2 = np.sum(np.asarray(q, np.float64) ** 2, axis=-1) * np.asarray(s, np.float64) ** 2
    meta = np.zeros(np.shape(s) + (4,), np.float32)
    meta[..., 0] = s
    meta[..., 1] = n2
    assert np.array_equal(meta[..., 1].astype(np.float64), n2), "squared norm not exact in fp32"
    return meta


def pack_rows(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """The stored rows, int8 [..., 144]: q, then the record's 16 bytes."""
    meta = row_meta(q, s)
    out = np.zeros(np.shape(q)[:-1] + (144,), np.int8)
    out[..., :128] = q
    out[..., 128:] = meta.view(np.int8).reshape(np.shape(q)[:-1] + (16,))
    return out


def dequantize_bits(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """k~ = s q as bf16 bits [..., d]; raises if some value is not exactly a
    bf16 number (it always is for scales of normal magnitude: |q| < 2^7)."""
    v = np.asarray(q, np.float64) * np.asarray(s, np.float64)[..., None]
    f = v.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), v), "s q not exact in fp32"
    u = f.view(np.uint32)
    assert not np.any(u & 0xFFFF), "s q not exact in bf16"
    return (u >> 16).astype(np.uint16)

"""Conversions between the oracle's logical codes and the library's packed
code layouts (test infrastructure; no hashing arithmetic here).

Logical codes: uint16 [..., N, L] (the table-l code of token i).
Library layouts (include/magicpig.h):
  bytes (K = 8): uint8 [..., L, Ncap]
  planes (any K): uint32 bit planes [..., L, Ncap/32, K], bit t of word (w, b) = bit b of token 32 w + t.
By default K = 8 uses bytes and K = 10 planes.
"""
import numpy as np


def pack_codes(logical: np.ndarray, K: int, Ncap: int, planes=None) -> np.ndarray:
    """[..., N, L] uint16 -> the library layout with capacity Ncap (zero past N)."""
    planes = (K != 8) if planes is None else planes
    *lead, N, L = logical.shape
    full = np.zeros((*lead, Ncap, L), np.uint16)
    full[..., :N, :] = logical
    if not planes:
        return np.ascontiguousarray(np.swapaxes(full, -1, -2)).astype(np.uint8)
    bits = ((full[..., None] >> np.arange(K, dtype=np.uint16)) & 1).astype(np.uint8)  # [..., Ncap, L, K]
    bits = np.moveaxis(bits, -3, -1)  # [..., L, K, Ncap]
    packed = np.packbits(bits.reshape(*bits.shape[:-1], Ncap // 32, 32), axis=-1, bitorder="little")
    words = np.ascontiguousarray(packed).view("<u4")[..., 0].astype(np.uint32)  # [..., L, K, Ncap/32]
    return np.ascontiguousarray(np.swapaxes(words, -1, -2))  # [..., L, Ncap/32, K]


def unpack_codes(packed: np.ndarray, K: int, L: int, N: int, planes=None) -> np.ndarray:
    """Library layout -> logical uint16 [..., N, L] (first N tokens)."""
    planes = (K != 8) if planes is None else planes
    if not planes:
        return np.ascontiguousarray(np.swapaxes(packed[..., :N], -1, -2)).astype(np.uint16)
    words = np.ascontiguousarray(np.swapaxes(packed.astype(np.uint32), -1, -2))  # [..., L, K, W]
    bytes_ = words.view(np.uint8).reshape(*words.shape, 4)
    bits = np.unpackbits(bytes_, axis=-1, bitorder="little").reshape(*words.shape[:-1], -1)[..., :N]
    w = (1 << np.arange(K, dtype=np.uint32))[:, None]
    codes = (bits.astype(np.uint32) * w).sum(axis=-2)  # [..., L, N]
    return np.ascontiguousarray(np.swapaxes(codes, -1, -2)).astype(np.uint16)

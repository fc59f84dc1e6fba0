"""fp64 CPU oracle for MagicPIG LSH-sampled decode attention.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs are the only callers.
The product path never imports this package, and this package never imports
the product package: the two share nothing but the seeded input generator.

The arithmetic lives in ``magicpig_oracle.c`` (plain fp64 loops, one function
per method step, each citing the passage it follows).  This module compiles it
with gcc on first use (or via ``build()``) and marshals numpy arrays into it.
``brute.py`` is a second, independent pure-Python restatement used to pin the
C code on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "magicpig_oracle.c")
_LIB = os.path.join(_HERE, "libmagicpig_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
               "-fPIC", "-std=c11", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.mpo_simhash.argtypes = [P, ctypes.c_int64, I, P, I, I, P, P]
        lib.mpo_simhash.restype = None
        lib.mpo_collision_prob.argtypes = [P, P, I]
        lib.mpo_collision_prob.restype = ctypes.c_double
        lib.mpo_sampling_prob.argtypes = [ctypes.c_double, I, I]
        lib.mpo_sampling_prob.restype = ctypes.c_double
        lib.mpo_collide.argtypes = [P, P, I, I, I, I, I, P, P]
        lib.mpo_collide.restype = None
        lib.mpo_attend.argtypes = [P, P, P, I, I, P, I, I, I, I, P, P]
        lib.mpo_attend.restype = None
        lib.mpo_decode.argtypes = [P, P, P, P, P, P] + [I] * 9 + [P, P, P, P]
        lib.mpo_decode.restype = None
        lib.mpo_num_threads.argtypes = []
        lib.mpo_num_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns")
    return a


def num_threads() -> int:
    return int(_load().mpo_num_threads())


def simhash(x_bits: np.ndarray, W_bits: np.ndarray, K: int, L: int, margin: bool = False):
    """SimHash codes of rows ``x_bits`` [..., d] (bf16 bits) against hyperplanes
    ``W_bits`` [L*K, d].  Returns codes [..., L] (uint16) and, if asked, the
    relative margin |x.w| / (|x||w|) of every bit [..., L*K]."""
    x = _u16(x_bits)
    W = _u16(W_bits)
    d = x.shape[-1]
    assert W.shape == (L * K, d), W.shape
    n = int(np.prod(x.shape[:-1]))
    codes = np.zeros((n, L), np.uint16)
    mg = np.zeros((n, L * K), np.float64) if margin else None
    _load().mpo_simhash(_ptr(x), n, d, _ptr(W), K, L, _ptr(codes),
                        _ptr(mg) if margin else None)
    codes = codes.reshape(x.shape[:-1] + (L,))
    if margin:
        return codes, mg.reshape(x.shape[:-1] + (L * K,))
    return codes


def collision_prob(q: np.ndarray, k: np.ndarray) -> float:
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    return float(_load().mpo_collision_prob(_ptr(q), _ptr(k), q.shape[0]))


def sampling_prob(p: float, K: int, L: int) -> float:
    return float(_load().mpo_sampling_prob(float(p), int(K), int(L)))


def collide(kcodes: np.ndarray, qcodes: np.ndarray, sink: int, window: int):
    """Membership of S_h for one unit: kcodes [N, L], qcodes [G, L] ->
    member [G, N] (uint8), n_sampled [G] (int32)."""
    kc = np.ascontiguousarray(kcodes, np.uint16)
    qc = np.ascontiguousarray(qcodes, np.uint16)
    N, L = kc.shape
    G = qc.shape[0]
    member = np.zeros((G, N), np.uint8)
    n = np.zeros(G, np.int32)
    _load().mpo_collide(_ptr(kc), _ptr(qc), N, L, G, sink, window, _ptr(member), _ptr(n))
    return member, n


def attend(q_bits, K_bits, V_bits, member, sink: int, window: int, Kbits: int, L: int):
    """Estimator for one head: q [d], K/V [N, d] (bf16 bits), member [N]."""
    q = _u16(q_bits)
    Kr = _u16(K_bits)
    Vr = _u16(V_bits)
    N, d = Kr.shape
    m = np.ascontiguousarray(member, np.uint8)
    out = np.zeros(d, np.float64)
    lse = np.zeros(1, np.float64)
    _load().mpo_attend(_ptr(q), _ptr(Kr), _ptr(Vr), N, d, _ptr(m), sink, window, Kbits, L,
                       _ptr(out), _ptr(lse))
    return out, float(lse[0])


def decode(q_bits, K_bits, V_bits, kcodes, qcodes, seq_lens, *, Kbits: int, L: int,
           sink: int, window: int, want_member: bool = False):
    """One decode step for a batch given the codes.

    q [B, Hq, d]; K, V [B, Hkv, Ncap, d] (bf16 bits); kcodes [B, Hkv, Ncap, L];
    qcodes [B, Hq, L]; seq_lens [B].  Returns out [B, Hq, d] (fp64),
    lse [B, Hq], n_sampled [B, Hq] and, if asked, member [B, Hq, Ncap]."""
    q = _u16(q_bits)
    Kc = _u16(K_bits)
    Vc = _u16(V_bits)
    B, Hq, d = q.shape
    _, Hkv, Ncap, _ = Kc.shape
    kc = np.ascontiguousarray(kcodes, np.uint16)
    qc = np.ascontiguousarray(qcodes, np.uint16)
    assert kc.shape == (B, Hkv, Ncap, L) and qc.shape == (B, Hq, L)
    sl = np.ascontiguousarray(seq_lens, np.int32)
    out = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    ns = np.zeros((B, Hq), np.int32)
    mem = np.zeros((B, Hq, Ncap), np.uint8) if want_member else None
    _load().mpo_decode(_ptr(q), _ptr(Kc), _ptr(Vc), _ptr(kc), _ptr(qc), _ptr(sl),
                       B, Hq, Hkv, d, Ncap, Kbits, L, sink, window,
                       _ptr(mem) if want_member else None, _ptr(out), _ptr(lse), _ptr(ns))
    if want_member:
        return out, lse, ns, mem
    return out, lse, ns

"""Seeded synthetic inputs for LSH-sampled decode attention.

This module is shared by the CUDA library's tests/benchmark and by the fp64
oracle's tests.  It draws random numbers and rounds them to bf16; it holds none
of the method's arithmetic (no hashing, no collision test, no attention).

Every tensor of every (batch, kv head) unit comes from its own PCG64 stream,
keyed by (workload seed, tensor tag, b, kv head), so any single unit can be
regenerated on the host without regenerating the rest.

The workloads stand in for the long-context retrieval tasks (RULER on
Llama-3.1-8B) that the MagicPIG pages evaluate on: those prompts, the model and
its weights are not available, so the inputs are i.i.d. Gaussian keys, values
and queries with the Llama-3.1-8B attention shape (32 query / 8 kv heads,
head_dim 128) and a few planted "needle" keys aligned with the query.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "get", "make_inputs", "f32_to_bf16_bits", "bf16_bits_to_f32",
           "unit_keys_values", "round_capacity"]

_TAG_W, _TAG_Q, _TAG_K, _TAG_V, _TAG_PLANT, _TAG_POS, _TAG_LEN, _TAG_MU, _TAG_NEW = range(1, 10)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32)
    r = (u >> 16) & 1
    r += 0x7FFF
    r += u
    r >>= 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_capacity(n: int) -> int:
    """Token capacity: room for one appended token, rounded up to 128."""
    return ((n + 1 + 127) // 128) * 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    context: int                  # tokens per sequence (max length when ragged)
    k_bits: int
    n_tables: int
    sink: int = 4
    window: int = 64
    n_planted: int = 0            # needle keys per kv head
    plant: str = "random"         # "random" or "even" positions
    ragged_min: int = 0           # >0: lengths uniform in [ragged_min, context]
    mu_norm: float = 0.0          # >0: keys offset by a per-kv-head mean of this norm
    seed: int = 0
    description: str = ""
    code_layout: str = "auto"     # key-code layout: "auto", "bytes" (K = 8) or "planes"

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def capacity(self) -> int:
        return round_capacity(self.context)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload(
        "tiny", 1, 1, 1, 128, 2048, 8, 75, n_planted=16, seed=1001,
        description="single head, N=2048, K=8, L=75, sink 4 + window 64, 16 needles = q + 0.5 N(0,1)"),
    "llama8b_16k": Workload(
        "llama8b_16k", 1, 32, 8, 128, 16384, 8, 75, n_planted=32, seed=1002,
        description="Llama-3.1-8B-shaped layer (32 q / 8 kv heads), N=16384, K=8, L=75, "
                    "32 needles per kv head = mean of its q heads + 0.5 N(0,1)"),
    "batch8_64k": Workload(
        "batch8_64k", 8, 32, 8, 128, 65536, 10, 150, n_planted=64, plant="even", seed=1003,
        description="batch 8, N=65536, K=10, L=150 (bit-plane codes), 64 evenly spaced needles"),
    "batch4_128k": Workload(
        "batch4_128k", 4, 32, 8, 128, 131072, 10, 150, n_planted=64, plant="even", seed=1004,
        description="batch 4, N=131072, K=10, L=150; key hash build timed apart; one appended token"),
    "ragged16": Workload(
        "ragged16", 16, 32, 8, 128, 131072, 8, 75, n_planted=128, ragged_min=32768, mu_norm=8.0,
        seed=1005,
        description="batch 16, lengths U[32768,131072], K=8, L=75, keys = mu_h (|mu_h|=8) + N(0,1), "
                    "128 needles per kv head"),
    "ragged4": Workload(
        "ragged4", 4, 32, 8, 128, 131072, 8, 75, n_planted=128, ragged_min=32768, mu_norm=8.0,
        seed=1006,
        description="the ragged workload at batch 4 (about 2 GB of cache): the profiling case for the "
                    "K=8 scan and the sampled-attention kernel"),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


def seq_lens_of(w: Workload) -> np.ndarray:
    if w.ragged_min > 0:
        return _rng(w.seed, _TAG_LEN).integers(w.ragged_min, w.context + 1, size=w.batch).astype(np.int32)
    return np.full(w.batch, w.context, np.int32)


def hyperplanes_of(w: Workload) -> np.ndarray:
    """W: L*K hyperplanes of dimension d, drawn fp32 N(0,1) and rounded to bf16.
    Row c = l*K + b is the hyperplane of bit b of table l.  [L*K, d] uint16."""
    g = _rng(w.seed, _TAG_W)
    return f32_to_bf16_bits(g.standard_normal((w.n_tables * w.k_bits, w.head_dim), np.float32))


def queries_of(w: Workload) -> np.ndarray:
    g = _rng(w.seed, _TAG_Q)
    return f32_to_bf16_bits(g.standard_normal((w.batch, w.n_q_heads, w.head_dim), np.float32))


def mu_of(w: Workload, kv_head: int) -> Optional[np.ndarray]:
    if w.mu_norm <= 0:
        return None
    g = _rng(w.seed, _TAG_MU, kv_head)
    m = g.standard_normal(w.head_dim).astype(np.float64)
    return (m * (w.mu_norm / np.linalg.norm(m))).astype(np.float32)


def planted_positions(w: Workload, b: int, kv_head: int, n: int) -> np.ndarray:
    lo, hi = w.sink, n - w.window
    cnt = min(w.n_planted, max(0, hi - lo))
    if cnt <= 0:
        return np.zeros(0, np.int64)
    if w.plant == "even":
        return lo + ((np.arange(cnt) + 0.5) * (hi - lo) / cnt).astype(np.int64)
    g = _rng(w.seed, _TAG_POS, b, kv_head)
    return np.sort(g.choice(hi - lo, size=cnt, replace=False) + lo)


def unit_keys_values(w: Workload, q_bits: np.ndarray, b: int, kv_head: int, n: int):
    """Keys and values [n, d] (bf16 bits) of one (b, kv head) unit."""
    d = w.head_dim
    k = _rng(w.seed, _TAG_K, b, kv_head).standard_normal((n, d), np.float32)
    mu = mu_of(w, kv_head)
    if mu is not None:
        k += mu
    pos = planted_positions(w, b, kv_head, n)
    if len(pos):
        G = w.group
        qf = bf16_bits_to_f32(q_bits[b, kv_head * G:(kv_head + 1) * G]).astype(np.float32)
        centre = qf.mean(axis=0)
        noise = _rng(w.seed, _TAG_PLANT, b, kv_head).standard_normal((len(pos), d), np.float32)
        k[pos] = centre + np.float32(0.5) * noise
    v = _rng(w.seed, _TAG_V, b, kv_head).standard_normal((n, d), np.float32)
    return f32_to_bf16_bits(k), f32_to_bf16_bits(v)


def new_token_of(w: Workload):
    """One appended token per sequence: k_new, v_new [B, Hkv, d] (bf16 bits)."""
    g = _rng(w.seed, _TAG_NEW)
    shape = (w.batch, w.n_kv_heads, w.head_dim)
    return (f32_to_bf16_bits(g.standard_normal(shape, np.float32)),
            f32_to_bf16_bits(g.standard_normal(shape, np.float32)))


def make_inputs(w: Workload, threads: Optional[int] = None):
    """All inputs of one decode step.

    Returns a dict: W [L*K, d], q [B, Hq, d], K/V [B, Hkv, Ncap, d] (uint16 bf16
    bits; rows at and past each sequence length are zero), seq_lens [B] int32,
    k_new / v_new [B, Hkv, d]."""
    B, Hkv, d, cap = w.batch, w.n_kv_heads, w.head_dim, w.capacity
    W = hyperplanes_of(w)
    q = queries_of(w)
    lens = seq_lens_of(w)
    K = np.zeros((B, Hkv, cap, d), np.uint16)
    V = np.zeros((B, Hkv, cap, d), np.uint16)

    def fill(bk):
        b, kh = bk
        n = int(lens[b])
        K[b, kh, :n], V[b, kh, :n] = unit_keys_values(w, q, b, kh, n)

    units = [(b, kh) for b in range(B) for kh in range(Hkv)]
    nthreads = threads or min(len(units), os.cpu_count() or 1)
    if nthreads > 1:
        with ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(fill, units))
    else:
        for u in units:
            fill(u)
    k_new, v_new = new_token_of(w)
    return dict(W=W, q=q, K=K, V=V, seq_lens=lens, k_new=k_new, v_new=v_new)

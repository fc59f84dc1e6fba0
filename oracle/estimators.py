"""Baseline estimators of one decode head's attention output (CPU, fp64).

EVALUATION / TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: it puts
the error of MagicPIG's sampling estimate next to the two baselines the
MagicPIG project pages name among their prediction backends ("TopK baseline"
and "Oracle sampling", gitdiagram project page, "Prediction Backends"), on the
synthetic workloads.  The pages name these baselines but do not define them;
the readings below are the plainest ones consistent with the method:

* exact:   o = sum_i softmax(s)_i v_i over all N tokens, s_i = q.k_i / sqrt(d).
* TopK(k): the exact set D plus the k tokens outside D with the largest s_i,
  with the softmax renormalised over the kept tokens (a deterministic sparse
  approximation; it is biased whenever the attention is not sparse).
* oracle sampling(b): D exactly, plus b tokens drawn i.i.d. from the tokens
  outside D with probability proportional to exp(s_i) -- the ideal proposal,
  which needs the exact attention weights (hence "oracle").  With importance
  weights w_i / p_i = Z_S (Z_S = sum_{i not in D} exp(s_i)) the estimate is
  o = (sum_D w v + Z_S mean_j v_{i_j}) / (sum_D w + Z_S), unbiased for o.

All inputs are float64 arrays; scores are max-shifted before exponentiation.
"""
from __future__ import annotations

import numpy as np


def exact_set(n: int, sink: int, window: int) -> np.ndarray:
    """Boolean mask of D = [0, sink) U [n - window, n) over n tokens."""
    d = np.zeros(n, bool)
    d[:min(sink, n)] = True
    d[max(0, n - window):] = True
    return d


def scores(q: np.ndarray, K: np.ndarray) -> np.ndarray:
    return K @ q / np.sqrt(q.shape[0])


def exact_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    s = scores(q, K)
    w = np.exp(s - s.max())
    return w @ V / w.sum()


def topk_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, k: int, sink: int, window: int) -> np.ndarray:
    """Softmax attention restricted to D plus the top-k scored tokens outside D."""
    s = scores(q, K)
    n = s.shape[0]
    keep = exact_set(n, sink, window)
    rest = np.flatnonzero(~keep)
    if k > 0 and rest.size:
        top = rest[np.argsort(-s[rest], kind="stable")[:k]]
        keep[top] = True
    sk = s[keep]
    w = np.exp(sk - sk.max())
    return w @ V[keep] / w.sum()


def oracle_sampling(q: np.ndarray, K: np.ndarray, V: np.ndarray, budget: int, sink: int, window: int,
                    rng: np.random.Generator) -> np.ndarray:
    """D exactly plus `budget` i.i.d. draws from softmax(s) over the rest."""
    s = scores(q, K)
    n = s.shape[0]
    d = exact_set(n, sink, window)
    m = s.max()
    w = np.exp(s - m)
    num = w[d] @ V[d]
    den = w[d].sum()
    rest = np.flatnonzero(~d)
    if rest.size == 0 or budget <= 0:
        return num / den
    ws = w[rest]
    zs = ws.sum()
    pick = rng.choice(rest.size, size=budget, replace=True, p=ws / zs)
    return (num + zs * V[rest[pick]].mean(axis=0)) / (den + zs)


def rel_l2(x: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(x - ref) / np.linalg.norm(ref))

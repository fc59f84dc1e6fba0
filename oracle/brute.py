"""Second, independent restatement of the method in pure Python (tiny inputs).

TEST INFRASTRUCTURE ONLY.  Written separately from ``magicpig_oracle.c`` so
that the two pin each other: plain Python floats (IEEE fp64), ``math.comb``
for the binomial law and no numpy arithmetic.  Inputs are lists of floats
(already widened from bf16).  Follows the same method steps (MagicPIG, Chen et
al. 2024: SimHash codes, at-least-two-of-L collision sampling, importance
weights 1/u, exact sink and local-window set).
"""
from __future__ import annotations

import math


def simhash_code(x, W, K, L):
    """Codes of one vector: table l's code has bit b set iff x . W[l*K+b] > 0."""
    codes = []
    for l in range(L):
        c = 0
        for b in range(K):
            w = W[l * K + b]
            proj = math.fsum(xi * wi for xi, wi in zip(x, w))
            if proj > 0.0:
                c += 2 ** b
        codes.append(c)
    return codes


def angle_prob(q, k):
    """Per-bit collision probability of random-hyperplane hashing: 1 - theta/pi."""
    qq = math.sqrt(math.fsum(v * v for v in q))
    kk = math.sqrt(math.fsum(v * v for v in k))
    if qq == 0.0 or kk == 0.0:
        return 0.5
    c = math.fsum(a * b for a, b in zip(q, k)) / (qq * kk)
    c = min(1.0, max(-1.0, c))
    return 1.0 - math.acos(c) / math.pi


def at_least_two_of(L, x):
    """P[Binomial(L, x) >= 2] written as 1 - P[0] - P[1]."""
    if L < 2:
        return 0.0
    p0 = (1.0 - x) ** L
    p1 = L * x * (1.0 - x) ** (L - 1)
    return 1.0 - p0 - p1


def at_least_two_of_sum(L, x):
    """The same probability as an explicit binomial sum (for small u)."""
    return math.fsum(math.comb(L, j) * x ** j * (1.0 - x) ** (L - j) for j in range(2, L + 1))


def decode_head(q, keys, vals, W, K, L, sink, window):
    """Estimate for one query head over N tokens.  Returns (out, lse, S)."""
    N = len(keys)
    d = len(q)
    qc = simhash_code(q, W, K, L)
    exact = set(range(min(sink, N))) | set(range(max(0, N - window), N))
    S = []
    for i in range(N):
        if i in exact:
            continue
        kc = simhash_code(keys[i], W, K, L)
        if sum(1 for a, b in zip(kc, qc) if a == b) >= 2:
            S.append(i)
    logw = {}
    for i in sorted(exact) + S:
        s = math.fsum(a * b for a, b in zip(q, keys[i])) / math.sqrt(d)
        if i in exact:
            logw[i] = s
        else:
            x = angle_prob(q, keys[i]) ** K
            u = at_least_two_of_sum(L, x)
            logw[i] = s - math.log(u)
    if not logw:
        return [0.0] * d, -math.inf, S
    m = max(logw.values())
    wts = {i: math.exp(v - m) for i, v in logw.items()}
    z = math.fsum(wts.values())
    out = [math.fsum(wts[i] * vals[i][j] for i in wts) / z for j in range(d)]
    return out, m + math.log(z), S

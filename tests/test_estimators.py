"""Pins of the CPU baseline estimators (oracle/estimators.py) that the
estimator comparison puts next to MagicPIG: each is checked against a closed
form or a limit that fixes it, not against itself."""
import numpy as np
import pytest

from oracle import estimators as est


def _rand(n, d=16, seed=0):
    g = np.random.default_rng(seed)
    return g.standard_normal(d), g.standard_normal((n, d)), g.standard_normal((n, d))


def test_exact_attention_two_tokens_by_hand():
    q = np.array([1.0, 0.0, 0.0, 0.0])
    K = np.array([[2.0, 0, 0, 0], [0.0, 1, 0, 0]])
    V = np.array([[1.0, 0, 0, 0], [0.0, 1, 0, 0]])
    s1, s2 = 2.0 / 2.0, 0.0  # q.k / sqrt(4)
    a = np.exp(s1) / (np.exp(s1) + np.exp(s2))
    np.testing.assert_allclose(est.exact_attention(q, K, V), [a, 1 - a, 0, 0], rtol=1e-15)


def test_topk_with_every_token_is_exact():
    q, K, V = _rand(200)
    np.testing.assert_allclose(est.topk_attention(q, K, V, 200, 4, 16), est.exact_attention(q, K, V), rtol=1e-12)


def test_topk_zero_keeps_only_the_exact_set():
    q, K, V = _rand(100, seed=1)
    d = est.exact_set(100, 4, 16)
    np.testing.assert_allclose(est.topk_attention(q, K, V, 0, 4, 16), est.exact_attention(q, K[d], V[d]),
                               rtol=1e-12)


def test_topk_picks_the_highest_scores():
    q, K, V = _rand(64, seed=2)
    s = est.scores(q, K)
    d = est.exact_set(64, 2, 2)
    rest = np.flatnonzero(~d)
    top = rest[np.argsort(-s[rest])[:5]]
    keep = d.copy()
    keep[top] = True
    np.testing.assert_allclose(est.topk_attention(q, K, V, 5, 2, 2), est.exact_attention(q, K[keep], V[keep]),
                               rtol=1e-12)


def test_oracle_sampling_is_unbiased():
    """The mean of many oracle-sampling estimates converges to exact attention
    (each coordinate within 5 standard errors)."""
    q, K, V = _rand(40, d=8, seed=3)
    rng = np.random.default_rng(4)
    draws = np.array([est.oracle_sampling(q, K, V, 3, 2, 2, rng) for _ in range(20000)])
    ref = est.exact_attention(q, K, V)
    se = draws.std(axis=0) / np.sqrt(len(draws))
    assert (np.abs(draws.mean(axis=0) - ref) <= 5 * se + 1e-12).all()


def test_oracle_sampling_without_samples_is_the_exact_set():
    q, K, V = _rand(50, seed=5)
    d = est.exact_set(50, 4, 8)
    np.testing.assert_allclose(est.oracle_sampling(q, K, V, 0, 4, 8, np.random.default_rng(0)),
                               est.exact_attention(q, K[d], V[d]), rtol=1e-12)


def test_comparison_runs_on_the_single_head_workload():
    """On the single-head workload, whose needles are aligned with the query,
    MagicPIG's sample holds every needle and its estimate is close to exact."""
    from oracle.compare_estimators import compare, summary
    w, rows = compare("tiny", 1)
    s = summary(rows)
    assert s["needle_recall"]["magicpig"] == 1.0
    assert s["magicpig"]["mean_rel_l2"] < 1e-2
    assert 0 < s["budget_fraction"] < 0.5


def test_budget_grows_with_tables_and_shrinks_with_bits():
    """The sampling probability u = P[Bin(L, p^K) >= 2] grows with the number
    of tables L and falls with the bits per table K, and so must MagicPIG's
    budget |S_h| on the same keys (the codes of the first L' tables are the
    same for every L >= L' only in distribution, so the check is on the
    spread-out grid points)."""
    from oracle.compare_estimators import sweep
    r = sweep("tiny", 1, ks=(6, 10), ls=(25, 200))
    b = {kl: v["budget_fraction"] for kl, v in r.items()}
    assert b[(6, 200)] > b[(6, 25)] and b[(10, 200)] > b[(10, 25)]
    assert b[(6, 25)] > b[(10, 25)] and b[(6, 200)] > b[(10, 200)]
    # needles are q + small noise: every setting keeps them
    assert all(v["needle_recall"]["magicpig"] == 1.0 for v in r.values())

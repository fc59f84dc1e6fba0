"""Pins for the fp64 oracle, against what the method and the mathematics fix.

P1  per-table SimHash collision rate = (1 - theta/pi)^K (Monte Carlo over W)
P2  rate of "at least 2 of L tables collide" = u (Monte Carlo over W)
P3  the 1/u-weighted sums are unbiased for the exact sums (Monte Carlo over W)
P4  K = 0 (every table collides, u = 1): the estimator is exact softmax attention
P5  agreement with an independent pure-Python restatement on N <= 16
P6  stable binomial tail = closed form 1 - (1-x)^L - L x (1-x)^(L-1)
plus hand-derived golden values (tests/golden) for the sign/tie rule and u.
"""
import json
import math
import os

import numpy as np
import pytest

from workloads import bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf(a):
    return f32_to_bf16_bits(np.asarray(a, np.float32))


def _pair_at_angle(theta, d=128, scale=4.0):
    """q, k (bf16 bits) in a random 2-D plane at angle ~theta; returns the
    exact angle of the rounded vectors too."""
    rng = np.random.default_rng(int(theta * 1e6) + 7)
    basis, _ = np.linalg.qr(rng.standard_normal((d, 2)))
    q = scale * basis[:, 0]
    k = scale * (math.cos(theta) * basis[:, 0] + math.sin(theta) * basis[:, 1])
    qb, kb = _bf(q), _bf(k)
    qf = bf16_bits_to_f32(qb).astype(np.float64)
    kf = bf16_bits_to_f32(kb).astype(np.float64)
    c = np.clip(qf @ kf / np.linalg.norm(qf) / np.linalg.norm(kf), -1, 1)
    return qb, kb, math.acos(c)


def _gauss_W(rows, d, seed):
    return _bf(np.random.default_rng(seed).standard_normal((rows, d), np.float32))


# ---------------------------------------------------------------- golden ----

def test_golden_sign_rule_ties(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "simhash_ties.json")))
    codes = oracle_mod.simhash(_bf(g["keys"]), _bf(g["W"]), g["K"], g["L"])
    assert codes.tolist() == g["codes"]


def test_golden_sampling_prob(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "sampling_prob.json")))
    for e in g["u"]:
        assert oracle_mod.sampling_prob(e["p"], e["K"], e["L"]) == pytest.approx(e["u"], abs=1e-15), e
    for e in g["angle"]:
        t = math.radians(e["theta_deg"])
        q = np.zeros(8)
        q[0] = 1.0
        k = np.zeros(8)
        k[0], k[1] = math.cos(t), math.sin(t)
        assert oracle_mod.collision_prob(q, k) == pytest.approx(e["p"], abs=1e-12), e


def test_zero_vector_collision_prob_is_half(oracle_mod):
    assert oracle_mod.collision_prob(np.zeros(4), np.ones(4)) == 0.5


# -------------------------------------------------------------------- P1 ----

@pytest.mark.parametrize("theta_deg,K", [(20, 8), (45, 4), (70, 2), (110, 1), (60, 10)])
def test_p1_per_table_collision_rate(oracle_mod, theta_deg, K):
    L = 20000
    qb, kb, theta = _pair_at_angle(math.radians(theta_deg))
    W = _gauss_W(L * K, 128, seed=100 + theta_deg * 10 + K)
    codes = oracle_mod.simhash(np.stack([qb, kb]), W, K, L)
    rate = float(np.mean(codes[0] == codes[1]))
    expect = (1.0 - theta / math.pi) ** K
    sigma = math.sqrt(expect * (1 - expect) / L)
    assert abs(rate - expect) <= 4 * sigma + 1e-12, (rate, expect, sigma)


# -------------------------------------------------------------------- P2 ----

@pytest.mark.parametrize("theta_deg,K,L", [(68, 8, 75), (74, 8, 75), (64, 10, 150), (70, 10, 150), (72, 4, 12)])
def test_p2_at_least_two_of_L_rate_is_u(oracle_mod, theta_deg, K, L):
    trials = 3000
    qb, kb, theta = _pair_at_angle(math.radians(theta_deg), d=16)  # rate depends on angle only
    W = _gauss_W(trials * L * K, 16, seed=7 + theta_deg)
    codes = oracle_mod.simhash(np.stack([qb, kb]), W, K, trials * L)
    hits = (codes[0] == codes[1]).reshape(trials, L).sum(axis=1)
    rate = float(np.mean(hits >= 2))
    p = 1.0 - theta / math.pi
    u = oracle_mod.sampling_prob(p, K, L)
    sigma = math.sqrt(max(u * (1 - u), 1e-4) / trials)
    assert 0.05 < u < 0.95, u  # the chosen angles exercise the middle of the curve
    assert abs(rate - u) <= 4 * sigma, (rate, u, sigma)


# -------------------------------------------------------------------- P3 ----

def test_p3_importance_weights_are_unbiased(oracle_mod):
    """E over W of sum_{i in S} e^{s_i}/u_i v_i equals sum_i e^{s_i} v_i (D empty),
    and likewise for the normaliser: inclusion in S has probability exactly u_i."""
    K, L, d, trials = 4, 10, 128, 3000
    rng = np.random.default_rng(5)
    angles = [0.35, 0.55, 0.75, 0.95, 1.2]
    q = _bf(rng.standard_normal(d))
    qf = bf16_bits_to_f32(q).astype(np.float64)
    qn = qf / np.linalg.norm(qf)
    keys = []
    for a in angles:
        r = rng.standard_normal(d)
        r -= (r @ qn) * qn
        r /= np.linalg.norm(r)
        keys.append(_bf(3.0 * (math.cos(a) * qn + math.sin(a) * r)))
    keys = np.stack(keys)
    vals = _bf(rng.standard_normal((len(angles), d)))
    kf = bf16_bits_to_f32(keys).astype(np.float64)
    vf = bf16_bits_to_f32(vals).astype(np.float64)
    s = kf @ qf / math.sqrt(d)
    exact_num = (np.exp(s)[:, None] * vf).sum(axis=0)
    exact_den = np.exp(s).sum()
    nums, dens = [], []
    for t in range(trials):
        W = _gauss_W(L * K, d, seed=10_000 + t)
        codes = oracle_mod.simhash(np.concatenate([q[None], keys]), W, K, L)
        member, _ = oracle_mod.collide(codes[1:], codes[:1], sink=0, window=0)
        out, lse = oracle_mod.attend(q, keys, vals, member[0], 0, 0, K, L)
        if lse == -math.inf:
            nums.append(np.zeros(d))
            dens.append(0.0)
        else:
            z = math.exp(lse)
            nums.append(out * z)
            dens.append(z)
    nums = np.array(nums)
    dens = np.array(dens)
    se_den = dens.std(ddof=1) / math.sqrt(trials)
    assert abs(dens.mean() - exact_den) <= 4 * se_den, (dens.mean(), exact_den, se_den)
    se_num = nums.std(axis=0, ddof=1) / math.sqrt(trials)
    z = np.abs(nums.mean(axis=0) - exact_num) / se_num
    assert np.mean(z <= 4) >= 0.99 and z.max() < 6, z.max()


# -------------------------------------------------------------------- P4 ----

@pytest.mark.parametrize("sink,window", [(0, 0), (4, 64), (200, 200)])
def test_p4_all_sampled_limit_is_exact_softmax(oracle_mod, sink, window):
    """K = 0: every code is empty, all L tables collide, u = 1 for L >= 2, so
    the estimator is exact softmax attention over the whole context."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, d, N, L = 2, 4, 2, 128, 300, 5
    q = _bf(rng.standard_normal((B, Hq, d)))
    Kc = _bf(rng.standard_normal((B, Hkv, N, d)))
    Vc = _bf(rng.standard_normal((B, Hkv, N, d)))
    W = np.zeros((0, d), np.uint16)
    kcodes = oracle_mod.simhash(Kc, W, 0, L)
    qcodes = oracle_mod.simhash(q, W, 0, L)
    lens = np.array([N, N - 37], np.int32)
    out, lse, ns = oracle_mod.decode(q, Kc, Vc, kcodes, qcodes, lens, Kbits=0, L=L,
                                     sink=sink, window=window)
    qf, kf, vf = (bf16_bits_to_f32(a).astype(np.float64) for a in (q, Kc, Vc))
    G = Hq // Hkv
    for b in range(B):
        n = lens[b]
        for h in range(Hq):
            s = kf[b, h // G, :n] @ qf[b, h] / math.sqrt(d)
            m = s.max()
            e = np.exp(s - m)
            ref = (e[:, None] * vf[b, h // G, :n]).sum(0) / e.sum()
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-12, atol=1e-13)
            assert lse[b, h] == pytest.approx(m + math.log(e.sum()), rel=1e-13)
            n_exact = len(set(range(min(sink, n))) | set(range(max(0, n - window), n)))
            assert ns[b, h] == n - n_exact


# -------------------------------------------------------------------- P5 ----

@pytest.mark.parametrize("seed,N,K,L,sink,window", [
    (0, 16, 2, 6, 1, 2), (1, 12, 3, 8, 0, 0), (2, 9, 1, 4, 2, 1), (3, 16, 2, 6, 20, 0), (4, 5, 2, 3, 1, 1)])
def test_p5_brute_force_agreement(oracle_mod, seed, N, K, L, sink, window):
    from oracle import brute
    rng = np.random.default_rng(seed)
    d = 16
    q = _bf(rng.standard_normal(d))
    keys = rng.standard_normal((N, d))
    keys[: N // 3] = bf16_bits_to_f32(q) + 0.4 * keys[: N // 3]  # some near-duplicates
    keys = _bf(keys)
    vals = _bf(rng.standard_normal((N, d)))
    W = _bf(rng.standard_normal((L * K, d)))
    Wf = bf16_bits_to_f32(W).astype(np.float64).tolist()
    qf = bf16_bits_to_f32(q).astype(np.float64).tolist()
    kf = bf16_bits_to_f32(keys).astype(np.float64).tolist()
    vf = bf16_bits_to_f32(vals).astype(np.float64).tolist()
    ref_out, ref_lse, ref_S = brute.decode_head(qf, kf, vf, Wf, K, L, sink, window)
    kc = oracle_mod.simhash(keys, W, K, L)
    qc = oracle_mod.simhash(q[None], W, K, L)
    assert kc.tolist() == [brute.simhash_code(k, Wf, K, L) for k in kf]
    assert qc[0].tolist() == brute.simhash_code(qf, Wf, K, L)
    member, ns = oracle_mod.collide(kc, qc, sink, window)
    assert np.flatnonzero(member[0]).tolist() == ref_S
    assert ns[0] == len(ref_S)
    out, lse = oracle_mod.attend(q, keys, vals, member[0], sink, window, K, L)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-13)
    assert lse == pytest.approx(ref_lse, rel=1e-12, abs=1e-13)


def test_p5_sampling_prob_matches_brute(oracle_mod):
    from oracle import brute
    for K, L in [(1, 2), (2, 7), (8, 75), (10, 150)]:
        for p in np.linspace(0.05, 0.999, 23):
            x = p ** K
            assert oracle_mod.sampling_prob(p, K, L) == pytest.approx(
                brute.at_least_two_of_sum(L, x), rel=1e-12, abs=1e-300)


# -------------------------------------------------------------------- P6 ----

@pytest.mark.parametrize("K,L", [(1, 2), (2, 3), (8, 75), (10, 150), (8, 200)])
def test_p6_tail_sum_matches_closed_form(oracle_mod, K, L):
    from oracle import brute
    checked = 0
    for p in np.linspace(0.0, 1.0, 401):
        u = oracle_mod.sampling_prob(p, K, L)
        assert 0.0 <= u <= 1.0
        closed = brute.at_least_two_of(L, p ** K)
        if closed > 1e-6:
            # the closed form loses ~eps/u to cancellation
            assert u == pytest.approx(closed, rel=1e-12 + 4e-16 * L / closed), (p, u, closed)
            checked += 1
    assert checked > 20


def test_u_is_monotone_in_p(oracle_mod):
    for K, L in [(8, 75), (10, 150)]:
        us = [oracle_mod.sampling_prob(p, K, L) for p in np.linspace(0, 1, 200)]
        assert all(b >= a - 1e-14 for a, b in zip(us, us[1:]))


# ----------------------------------------------------------- edge cases ----

def test_short_context_is_all_exact(oracle_mod):
    """N <= sink + window: D covers every token and S is empty."""
    rng = np.random.default_rng(3)
    N, d, K, L = 50, 128, 8, 75
    q = _bf(rng.standard_normal(d))
    keys = _bf(rng.standard_normal((N, d)))
    vals = _bf(rng.standard_normal((N, d)))
    member = np.ones(N, np.uint8)  # ignored inside D
    out, lse = oracle_mod.attend(q, keys, vals, member, 4, 64, K, L)
    qf, kf, vf = (bf16_bits_to_f32(a).astype(np.float64) for a in (q, keys, vals))
    s = kf @ qf / math.sqrt(d)
    e = np.exp(s - s.max())
    np.testing.assert_allclose(out, (e[:, None] * vf).sum(0) / e.sum(), rtol=1e-12)
    kc = oracle_mod.simhash(keys, _gauss_W(L * K, d, 1), K, L)
    mem, ns = oracle_mod.collide(kc, kc[:1], 4, 64)
    assert ns[0] == 0 and mem.sum() == 0


def test_empty_context(oracle_mod):
    out, lse = oracle_mod.attend(np.zeros(128, np.uint16), np.zeros((0, 128), np.uint16),
                                 np.zeros((0, 128), np.uint16), np.zeros(0, np.uint8), 4, 64, 8, 75)
    assert lse == -math.inf and not out.any()


def test_collide_excludes_exact_set_and_counts(oracle_mod):
    N, L = 40, 6
    kc = np.zeros((N, L), np.uint16)
    qc = np.zeros((2, L), np.uint16)
    qc[1] = 1  # head 1 matches nothing...
    kc[10, :2] = 1  # ...except token 10 in exactly two tables
    kc[11, :1] = 1  # and token 11 in one table only
    member, ns = oracle_mod.collide(kc, qc, sink=3, window=5)
    assert ns[0] == N - 8
    assert member[0, :3].sum() == 0 and member[0, -5:].sum() == 0
    assert np.flatnonzero(member[1]).tolist() == [10]

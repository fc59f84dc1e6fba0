"""Accuracy of MagicPIG's estimate next to TopK attention and oracle sampling.

EVALUATION INFRASTRUCTURE (CPU, fp64; see estimators.py for the readings of
the two baselines).  For a few (sequence, kv head) units of a synthetic
workload and every query head of the group it computes the exact attention
output and three estimates at the same token budget -- the number of sampled
tokens |S_h| that MagicPIG's LSH test selects for that head:

  magicpig        fp64 oracle of the method (SimHash codes, >= 2-of-L
                  collisions, weights exp(s - log u), exact set D)
  magicpig_int8   the same on the int8 keys s q of the library's opt-in
                  reduced-precision gather (oracle/kquant.py; same codes)
  topk            D plus the |S_h| highest-scored tokens, renormalised
  oracle_sampling D plus |S_h| i.i.d. draws from the exact softmax

and reports the relative L2 error against exact attention and the fraction
of planted needle keys each token set contains.

    python -m oracle.compare_estimators --workload llama8b_16k --units 2
    python -m oracle.compare_estimators --workload tiny --units 1 --sweep
"""
from __future__ import annotations

import argparse
import json

import numpy as np

from oracle import attend, build, collide, kquant, simhash
from oracle.estimators import exact_attention, oracle_sampling, rel_l2, scores, topk_attention, exact_set


def _f64(bits: np.ndarray) -> np.ndarray:
    from workloads import bf16_bits_to_f32
    return bf16_bits_to_f32(bits).astype(np.float64)


def compare_unit(w, q_bits, W_bits, b: int, kvh: int, n: int, rng: np.random.Generator, draws: int = 4):
    """Per-head rows for one unit: dicts of errors, budget and needle recall."""
    from workloads import planted_positions, unit_keys_values
    Kb, Vb = unit_keys_values(w, q_bits, b, kvh, n)
    G = w.group
    qh = q_bits[b, kvh * G:(kvh + 1) * G]
    kcodes = simhash(Kb, W_bits, w.k_bits, w.n_tables)
    qcodes = simhash(qh, W_bits, w.k_bits, w.n_tables)
    member, nsamp = collide(kcodes, qcodes, w.sink, w.window)
    K, V = _f64(Kb), _f64(Vb)
    q8, s8 = kquant.quantize_rows(Kb)
    Kt = kquant.dequantize_bits(q8, s8)
    needles = planted_positions(w, b, kvh, n)
    d = exact_set(n, w.sink, w.window)
    rows = []
    for g in range(G):
        q = _f64(qh[g])
        ref = exact_attention(q, K, V)
        mp_out, _ = attend(qh[g], Kb, Vb, member[g], w.sink, w.window, w.k_bits, w.n_tables)
        mp8_out, _ = attend(qh[g], Kt, Vb, member[g], w.sink, w.window, w.k_bits, w.n_tables)
        k = int(nsamp[g])
        tk = topk_attention(q, K, V, k, w.sink, w.window)
        osamp = [rel_l2(oracle_sampling(q, K, V, k, w.sink, w.window, rng), ref) for _ in range(draws)]
        s = scores(q, K)
        rest = np.flatnonzero(~d)
        top = set(rest[np.argsort(-s[rest], kind="stable")[:k]].tolist()) if k else set()
        nd = needles[~d[needles]] if len(needles) else needles
        rows.append(dict(
            budget=k, n=n,
            magicpig=rel_l2(mp_out, ref), magicpig_int8=rel_l2(mp8_out, ref), topk=rel_l2(tk, ref),
            oracle_sampling=float(np.mean(osamp)),
            recall_magicpig=float(member[g][nd].mean()) if len(nd) else float("nan"),
            recall_topk=float(np.mean([t in top for t in nd])) if len(nd) else float("nan")))
    return rows


def compare(name: str, units: int, seed: int = 0, **overrides):
    """Rows of compare_unit over `units` evenly picked units of workload
    `name` (fields replaced by `overrides`, e.g. k_bits, n_tables)."""
    import workloads
    w = workloads.get(name)
    if overrides:
        w = w.with_(**overrides)
    q_bits = workloads.queries_of(w)
    W_bits = workloads.hyperplanes_of(w)
    lens = workloads.seq_lens_of(w)
    rng = np.random.default_rng(seed)
    picks = [(b, kvh) for b in range(w.batch) for kvh in range(w.n_kv_heads)]
    pick_idx = np.linspace(0, len(picks) - 1, num=min(units, len(picks))).round().astype(int)
    rows = []
    for i in pick_idx:
        b, kvh = picks[i]
        rows += compare_unit(w, q_bits, W_bits, b, kvh, int(lens[b]), rng)
    return w, rows


def summary(rows):
    out = {}
    for m in ("magicpig", "magicpig_int8", "topk", "oracle_sampling"):
        v = np.array([r[m] for r in rows])
        out[m] = dict(mean_rel_l2=float(v.mean()), max_rel_l2=float(v.max()))
    out["budget_fraction"] = float(np.mean([r["budget"] / r["n"] for r in rows]))
    out["needle_recall"] = dict(magicpig=float(np.nanmean([r["recall_magicpig"] for r in rows])),
                                topk=float(np.nanmean([r["recall_topk"] for r in rows])))
    return out


SWEEP_K = (6, 8, 10)
SWEEP_L = (25, 50, 75, 100, 150, 200)


def sweep(name: str, units: int, seed: int = 0, ks=SWEEP_K, ls=SWEEP_L):
    """Budget, errors and needle recall of the three estimators over a grid
    of (K bits, L tables) on one workload: more tables sample more tokens,
    more bits per table fewer."""
    out = {}
    for K in ks:
        for L in ls:
            _, rows = compare(name, units, seed, k_bits=K, n_tables=L)
            out[(K, L)] = summary(rows)
    return out


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--workload", action="append", default=None)
    p.add_argument("--units", type=int, default=2)
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--sweep", action="store_true", help="grid over K in 6, 8, 10 and L in 25 .. 200")
    args = p.parse_args()
    build()
    res = {}
    for name in args.workload or ["tiny", "llama8b_16k"]:
        if args.sweep:
            print(f"{name}: K L budget/N magicpig topk oracle_sampling recall_magicpig recall_topk", flush=True)
            for (K, L), r in sweep(name, args.units, args.seed).items():
                print(f"{name}: {K} {L} {r['budget_fraction']:.4f} {r['magicpig']['mean_rel_l2']:.3g} "
                      f"{r['topk']['mean_rel_l2']:.3g} {r['oracle_sampling']['mean_rel_l2']:.3g} "
                      f"{r['needle_recall']['magicpig']:.2f} {r['needle_recall']['topk']:.2f}", flush=True)
                res[(name, K, L)] = r
            continue
        w, rows = compare(name, args.units, args.seed)
        res[name] = summary(rows)
        print(name, json.dumps(res[name]), flush=True)
    return res


if __name__ == "__main__":
    main()

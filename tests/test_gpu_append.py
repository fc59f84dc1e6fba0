"""The append kernel (one thread-block cluster per sequence, the length moved
by the same kernel): three calls in a row write each sequence's new K/V row
and code column at its current length and move the length by one each time;
a sequence at capacity is left as it is and reported; the appended codes
match the oracle within the near-zero tolerance.  Shapes cover one and many
kv heads, byte codes and bit planes, K = 8 and 10, and fewer tables than the
blocks of a cluster."""
import numpy as np
import pytest
import torch

from gpu_harness import Run, code_mismatch, dev, host, oracle_unit_codes
from workloads import WORKLOADS, f32_to_bf16_bits

import lsh_sampled_sparse_simhash_b200 as mp

pytestmark = pytest.mark.gpu

TINY = WORKLOADS["tiny"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()


CASES = {
    "g1_8kv_k8": dict(batch=5, n_q_heads=8, n_kv_heads=8, k_bits=8, n_tables=75, code_layout="auto"),
    "g4_k10": dict(batch=3, n_q_heads=8, n_kv_heads=2, k_bits=10, n_tables=150, code_layout="auto"),
    "g8_k8_planes": dict(batch=2, n_q_heads=16, n_kv_heads=2, k_bits=8, n_tables=75, code_layout="planes"),
    "few_tables": dict(batch=2, n_q_heads=4, n_kv_heads=1, k_bits=8, n_tables=5, code_layout="auto"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_three_appends_per_sequence(name):
    w = TINY.with_(name="app_" + name, context=700, n_planted=0, seed=2201, **CASES[name])
    run = Run(w)
    cap = w.capacity
    rng = np.random.default_rng(2202)
    # ragged start lengths; the last sequence is full (its appends must fail)
    start = rng.integers(0, cap - 3, size=w.batch).astype(np.int32)
    start[-1] = cap
    run.lens.copy_(torch.from_numpy(start))
    run.hash_keys(cap)  # every slot hashed once: the appends must overwrite their columns
    before_codes = [[run.codes_logical(b, kh, cap) for kh in range(w.n_kv_heads)] for b in range(w.batch)]
    before_k = host(run.K).view(np.uint16).copy()
    new_k, new_v = [], []
    for step in range(3):
        kf = rng.standard_normal((w.batch, w.n_kv_heads, 128)).astype(np.float32)
        vf = rng.standard_normal((w.batch, w.n_kv_heads, 128)).astype(np.float32)
        k_bits, v_bits = f32_to_bf16_bits(kf), f32_to_bf16_bits(vf)
        new_k.append(k_bits)
        new_v.append(v_bits)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        mp.append_token(run.shape, dev(k_bits), dev(v_bits), run.W, run.K, run.V, run.codes, run.lens, status)
        torch.cuda.synchronize()
        assert int(status.item()) == mp.MP_ERR_CAPACITY  # the full sequence
    lens = host(run.lens)
    K, V = host(run.K).view(np.uint16), host(run.V).view(np.uint16)
    for b in range(w.batch):
        if start[b] >= cap:
            assert lens[b] == start[b]
            np.testing.assert_array_equal(K[b], before_k[b])
            continue
        assert lens[b] == start[b] + 3
        for kh in range(w.n_kv_heads):
            got = run.codes_logical(b, kh, cap)
            for step in range(3):
                pos = start[b] + step
                np.testing.assert_array_equal(K[b, kh, pos], new_k[step][b, kh])
                np.testing.assert_array_equal(V[b, kh, pos], new_v[step][b, kh])
                ref, margin = oracle_unit_codes({"K": new_k[step][:, :, None], "W": run.inp["W"]}, w, b, kh, 1)
                bad, _ = code_mismatch(got[pos:pos + 1], ref, margin, w.k_bits)
                assert bad == 0, (b, kh, step)
            # every other token's code is untouched
            keep = np.ones(cap, bool)
            keep[start[b]:start[b] + 3] = False
            np.testing.assert_array_equal(got[keep], before_codes[b][kh][keep])

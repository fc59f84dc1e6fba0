"""The int8 key gather (mp_quantize_keys, mp_append_token_q8,
mp_decode_attend_q8) through the C ABI.

Bars:
  - the int8 rows and their scales bit-exact against the format's reference
    (oracle/kquant.py), rows outside the requested range untouched;
  - decode on the int8 copy against the fp64 oracle run on the dequantized keys
    s q with the same codes: candidate sets exact, out within 2e-3 relative L2
    and lse within 1e-3 (the bf16 path's own bars: the int8 path computes the
    same estimator on those keys);
  - the same decode against the oracle on the bf16 keys within the int8
    tolerance (2e-2 relative L2, 1e-2 on lse), the error the format costs.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import kquant
from gpu_harness import Run, check_outputs, host, oracle_decode_units, oracle_query_codes, oracle_unit_codes
from layout import unpack_codes
from test_kquant_oracle import INT8_REL_L2_TOL
from workloads import WORKLOADS, f32_to_bf16_bits, make_inputs

import lsh_sampled_sparse_simhash_b200 as mp

pytestmark = pytest.mark.gpu

INT8_LSE_ABS_TOL = 1e-2

TINY = WORKLOADS["tiny"]
CASES = {
    "tiny_g1_k8": TINY,
    "g4_k8_ragged_tail": TINY.with_(name="q8g4", batch=2, n_q_heads=8, n_kv_heads=2, context=5000,
                                    n_planted=16, seed=2101),
    "g8_k8_mu_offset": TINY.with_(name="q8g8", batch=1, n_q_heads=16, n_kv_heads=2, context=4100, mu_norm=8.0,
                                  n_planted=8, seed=2102),
    "g4_k10": TINY.with_(name="q8k10", batch=2, n_q_heads=8, n_kv_heads=2, context=9000, k_bits=10,
                         n_tables=150, n_planted=24, seed=2103),
    "g2_k8_planes": TINY.with_(name="q8p", batch=2, n_q_heads=4, n_kv_heads=2, context=3000, n_planted=8,
                               seed=2104, code_layout="planes"),
}


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()


def _plant_edge_rows(inp):
    """Rows that exercise the format's corners in unit (0, 0): a zero row, a
    row whose maximum is exactly 127 (scale 1, integer values: exact), one
    just above (128: scale 2, with halves that round to even) and a row of
    tiny values."""
    K = inp["K"]
    d = K.shape[-1]
    rows = np.zeros((4, d), np.float32)
    rows[1, :3] = [127.0, -1.0, 0.5]
    rows[2, :4] = [128.0, 3.0, -5.0, 1.0]
    rows[3] = np.linspace(-1e-3, 2e-3, d)
    K[0, 0, 5:9] = f32_to_bf16_bits(rows)


def _units(w):
    return [(b, kh) for b in range(w.batch) for kh in range(w.n_kv_heads)]


def _check_q8_rows(run, inp, units_rows):
    """Bit-exact 144-byte int8 rows (values and record) for {(b, kh): row indices}."""
    k8 = host(run.k8)
    for (b, kh), rows in units_rows.items():
        q, s = kquant.quantize_rows(inp["K"][b, kh, rows])
        np.testing.assert_array_equal(k8[b, kh, rows], kquant.pack_rows(q, s), err_msg=f"int8 rows b={b} kh={kh}")


def _meta(k8_rows):
    """The fp32 records of stored rows [..., 144]."""
    return np.ascontiguousarray(k8_rows[..., 128:]).view(np.float32)


@pytest.mark.parametrize("case", ["tiny_g1_k8", "g4_k8_ragged_tail", "g8_k8_mu_offset"])
def test_quantize_keys_bit_exact_and_bounded_by_lengths(case):
    w = CASES[case]
    inp = make_inputs(w)
    _plant_edge_rows(inp)
    run = Run(w, inp)
    run.alloc_q8()
    mp.quantize_keys(run.shape, run.K, run.k8, seq_lens=run.lens)
    torch.cuda.synchronize()
    lens = inp["seq_lens"]
    _check_q8_rows(run, inp, {(b, kh): np.arange(int(lens[b])) for b, kh in _units(w)})
    k8 = host(run.k8)
    km = _meta(k8)
    for b, kh in _units(w):
        n = int(lens[b])
        assert (k8[b, kh, n:] == 0x55).all(), "rows past the length written"
    assert list(km[0, 0, 5]) == [0.0, 0.0, 0.0, 0.0] and not k8[0, 0, 5].any()
    assert list(km[0, 0, 6]) == [1.0, 127.0 ** 2 + 1.0, 0.0, 0.0] and list(k8[0, 0, 6, :3]) == [127, -1, 0]
    assert list(km[0, 0, 7]) == [2.0, 4.0 * (64 ** 2 + 2 ** 2 + 2 ** 2), 0.0, 0.0]
    assert list(k8[0, 0, 7, :4]) == [64, 2, -2, 0]


def test_quantize_keys_token_range():
    """A sub-range [first_token, first_token + n) writes exactly those rows
    (a streamed prefill block)."""
    w = CASES["g4_k8_ragged_tail"]
    inp = make_inputs(w)
    run = Run(w, inp)
    run.alloc_q8()
    t0, n = 1000, 777
    mp.quantize_keys(run.shape, run.K, run.k8, first_token=t0, n_tokens=n)
    torch.cuda.synchronize()
    _check_q8_rows(run, inp, {u: np.arange(t0, t0 + n) for u in _units(w)})
    k8 = host(run.k8)
    assert (k8[:, :, :t0] == 0x55).all() and (k8[:, :, t0 + n:] == 0x55).all()


def _q8_run(w, inp):
    run = Run(w, inp)
    run.alloc_q8()
    mp.quantize_keys(run.shape, run.K, run.k8, seq_lens=run.lens)
    return run


def _dequantized(inp, units):
    out = {}
    for b, kh in units:
        n = int(inp["seq_lens"][b])
        q, s = kquant.quantize_rows(inp["K"][b, kh, :n])
        out[(b, kh)] = kquant.dequantize_bits(q, s)
    return out


def _decode_q8(w, edges):
    inp = make_inputs(w)
    if edges:
        _plant_edge_rows(inp)
    run = _q8_run(w, inp)
    units = _units(w)
    res = [oracle_unit_codes(inp, w, b, kh, int(inp["seq_lens"][b])) for b, kh in units]
    codes = [c for c, _ in res]
    run.set_codes(codes, units)
    qref, _ = oracle_query_codes(inp, w)
    gpu = run.decode(qcodes_in=qref, q8=True)
    assert gpu["status"] == 0
    return inp, units, codes, qref, gpu


@pytest.mark.parametrize("case", list(CASES))
def test_decode_q8_matches_oracle_on_dequantized_keys(case):
    """Same estimator as the oracle on the keys s q (codes from the bf16
    keys), with the format's corner rows planted in unit (0, 0)."""
    w = CASES[case]
    inp, units, codes, qref, gpu = _decode_q8(w, edges=True)
    ref = oracle_decode_units(inp, w, units, codes, qref, keys=_dequantized(inp, units))
    check_outputs(gpu, ref, w)


@pytest.mark.parametrize("case", ["g4_k8_ragged_tail", "g8_k8_mu_offset", "g4_k10"])
def test_decode_q8_error_against_bf16_keys(case):
    """What the format costs: the int8 decode against the oracle on the
    bf16 keys themselves."""
    w = CASES[case]
    inp, units, codes, qref, gpu = _decode_q8(w, edges=False)
    ref = oracle_decode_units(inp, w, units, codes, qref)
    worst = check_outputs(gpu, ref, w, rel_tol=INT8_REL_L2_TOL, lse_tol=INT8_LSE_ABS_TOL)
    print(f"{case}: int8 keys, worst rel-L2 {worst:.2e} against the bf16-key oracle")


def test_decode_q8_rejects_bf16_only_paths():
    w = CASES["g2_k8_planes"]
    run = _q8_run(w, make_inputs(w))
    for path in (mp.MP_PATH_FUSED, mp.MP_PATH_TC):
        with pytest.raises(mp.MagicPIGError):
            run.decode(path=path, q8=True)


def test_append_q8_writes_the_int8_row():
    """mp_append_token_q8 = mp_append_token plus the int8 row of each new key."""
    for w in (CASES["g4_k8_ragged_tail"], CASES["g4_k10"]):
        inp = make_inputs(w)
        run = _q8_run(w, inp)
        plain = Run(w, inp)
        run.hash_keys(w.context)
        plain.hash_keys(w.context)
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        mp.append_token_q8(run.shape, run.k_new, run.v_new, run.W, run.K, run.V, run.codes, run.lens, run.k8,
                           status[:1])
        mp.append_token(plain.shape, plain.k_new, plain.v_new, plain.W, plain.K, plain.V, plain.codes, plain.lens,
                        status[1:])
        torch.cuda.synchronize()
        assert host(status).tolist() == [0, 0]
        for a, c in ((run.K, plain.K), (run.V, plain.V), (run.codes, plain.codes), (run.lens, plain.lens)):
            assert torch.equal(a, c)
        pos = w.context
        k8 = host(run.k8)
        q, s = kquant.quantize_rows(inp["k_new"])
        np.testing.assert_array_equal(k8[:, :, pos], kquant.pack_rows(q, s))
        assert (k8[:, :, pos + 1:] == 0x55).all()


def test_append_q8_without_a_bf16_key_cache():
    """k_cache = NULL: the int8 row, the V row, the codes and the length are
    written as with a key cache, and the decode on the int8 copy is the same."""
    w = CASES["g4_k8_ragged_tail"]
    inp = make_inputs(w)
    run = _q8_run(w, inp)
    alt = _q8_run(w, inp)
    run.hash_keys(w.context)
    alt.hash_keys(w.context)
    run.alloc_decode(w.context + 1)
    alt.alloc_decode(w.context + 1)
    K_before = alt.K.clone()
    mp.append_token_q8(run.shape, run.k_new, run.v_new, run.W, run.K, run.V, run.codes, run.lens, run.k8)
    mp.append_token_q8(alt.shape, alt.k_new, alt.v_new, alt.W, None, alt.V, alt.codes, alt.lens, alt.k8)
    torch.cuda.synchronize()
    for a, c in ((run.V, alt.V), (run.codes, alt.codes), (run.lens, alt.lens), (run.k8, alt.k8)):
        assert torch.equal(a, c)
    assert torch.equal(alt.K, K_before)
    g1 = run.decode(q8=True)
    g2 = alt.decode(q8=True)
    np.testing.assert_array_equal(g1["member"], g2["member"])
    np.testing.assert_array_equal(g1["out"], g2["out"])


def test_full_size_q8_ragged16():
    """ragged16 in the benchmark's launch configuration with int8 keys:
    quantize the prefilled cache, append one token per sequence with its int8
    row, decode.  Every unit's candidate set against the oracle's collision
    rule on the same codes; the int8 rows of 512 sampled tokens and the
    appended token of every unit bit-exact; out / lse of 6 units spread over
    the length range against the oracle on the dequantized keys."""
    w = WORKLOADS["ragged16"]
    inp = make_inputs(w)
    run = Run(w, inp)
    run.alloc_q8()
    run.alloc_decode(run.max_len + 1)
    run.hash_keys(run.max_len)
    mp.quantize_keys(run.shape, run.K, run.k8, seq_lens=run.lens)
    mp.append_token_q8(run.shape, run.k_new, run.v_new, run.W, run.K, run.V, run.codes, run.lens, run.k8)
    torch.cuda.synchronize()
    new_lens = host(run.lens)
    assert (new_lens == inp["seq_lens"] + 1).all()
    for b in range(w.batch):
        inp["K"][b, :, inp["seq_lens"][b]] = inp["k_new"][b]
        inp["V"][b, :, inp["seq_lens"][b]] = inp["v_new"][b]
    inp["seq_lens"] = new_lens
    qref, _ = oracle_query_codes(inp, w)
    gpu = run.decode(qcodes_in=qref, q8=True)
    assert gpu["status"] == 0
    codes_h = host(run.codes)
    units = _units(w)
    order = sorted(units, key=lambda u: (int(new_lens[u[0]]), u))
    keep = {order[int(round(i * (len(order) - 1) / 5))] for i in range(6)}
    kept = {}
    rng = np.random.default_rng(1)
    G = w.group
    rows = {}
    for b, kh in units:
        n = int(new_lens[b])
        g = unpack_codes(codes_h[b, kh], w.k_bits, w.n_tables, n, run.shape.planes)
        hs = slice(kh * G, (kh + 1) * G)
        mem, ns = oracle.collide(g, qref[b, hs], w.sink, w.window)
        np.testing.assert_array_equal(gpu["member"][b, hs, :n], mem, err_msg=f"member b={b} kh={kh}")
        np.testing.assert_array_equal(gpu["ns"][b, hs], ns)
        rows[(b, kh)] = np.unique(np.concatenate([rng.choice(n - 1, size=512, replace=False), [n - 1]]))
        if (b, kh) in keep:
            kept[(b, kh)] = g
    _check_q8_rows(run, inp, rows)
    picked = sorted(kept)
    ref = oracle_decode_units(inp, w, picked, [kept[u] for u in picked], qref, keys=_dequantized(inp, picked))
    worst = check_outputs(gpu, ref, w)
    print(f"ragged16 int8 keys: {len(units)} units' candidate sets exact; worst rel-L2 {worst:.2e} over "
          f"{len(picked)} units against the oracle on s q keys")

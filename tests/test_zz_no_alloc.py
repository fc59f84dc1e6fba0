"""mp_decode_attend_noalloc: the decode entry point for callers that cannot
allocate device memory where they decode (a runtime with a memory pool sealed
after start-up, or a plugin that only receives tensors).  It must give
the same results as mp_decode_attend, which uses a caller-allocated workspace,
on consecutive calls that share the library's fixed scratch array.

Collected last (file name) so that a stop-at-first-failure run has already run
every other test; it builds everything it needs, so it also passes alone in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

REL_L2_TOL = 2e-3
LSE_ABS_TOL = 1e-3


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a)).cuda()


def _cases():
    from workloads import WORKLOADS
    tiny = WORKLOADS["tiny"]
    return {
        "llama8b_16k": WORKLOADS["llama8b_16k"],
        "k10_ragged": tiny.with_(name="k10r", batch=3, n_q_heads=8, n_kv_heads=2, context=9000, k_bits=10,
                                 n_tables=150, n_planted=16, seed=3001),
    }


@pytest.mark.parametrize("case", ["llama8b_16k", "k10_ragged"])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(case):
    import __graft_entry__
    __graft_entry__.build()
    import lsh_sampled_sparse_simhash_b200 as mp
    from workloads import make_inputs

    assert torch.cuda.is_available()
    w = _cases()[case]
    inp = make_inputs(w)
    if case == "k10_ragged":
        inp["seq_lens"] = np.array([9000, 4097, 70], np.int32)
    shape = mp.Shape(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.capacity, w.k_bits, w.n_tables,
                     w.sink, w.window)
    W, q, K, V = _dev(inp["W"]), _dev(inp["q"]), _dev(inp["K"]), _dev(inp["V"])
    lens = _dev(inp["seq_lens"].astype(np.int32))
    max_len = int(inp["seq_lens"].max())
    kind, cshape = mp.codes_shape(shape)
    codes = torch.zeros(cshape, dtype=torch.uint8 if kind == "uint8" else torch.int32, device="cuda")
    mp.hash_keys(shape, K, W, max_len, codes, seq_lens=lens)

    def outputs():
        return (torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device="cuda"),
                torch.empty((w.batch, w.n_q_heads), dtype=torch.float32, device="cuda"),
                torch.empty((w.batch, w.n_q_heads), dtype=torch.int32, device="cuda"))

    # reference: the workspace entry point
    ws = torch.empty(mp.decode_workspace_bytes(shape, max_len), dtype=torch.uint8, device="cuda")
    assert ws.numel() <= 16 << 20
    ref_out, ref_lse, ref_ns = outputs()
    mp.decode_attend(shape, q, W, codes, K, V, lens, max_len, ref_out, ref_lse, ref_ns, ws)
    torch.cuda.synchronize()
    assert mp.read_status(ws) == 0

    lib = mp.library()
    cs = shape.c()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):  # consecutive calls share (and inherit) the scratch contents
        out, lse, ns = outputs()
        status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
        rc = lib.mp_decode_attend_noalloc(ctypes.byref(cs), q.data_ptr(), W.data_ptr(), codes.data_ptr(),
                                          K.data_ptr(), V.data_ptr(), lens.data_ptr(), max_len, out.data_ptr(),
                                          lse.data_ptr(), ns.data_ptr(), status.data_ptr(), stream)
        assert rc == mp.MP_OK, mp.status_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == mp.MP_OK, f"call {call}"
        assert torch.equal(ns, ref_ns), f"call {call}: n_sampled differs"
        o, r = out.double().cpu().numpy(), ref_out.double().cpu().numpy()
        l, rl = lse.cpu().numpy(), ref_lse.cpu().numpy()
        for b in range(w.batch):
            for h in range(w.n_q_heads):
                if np.isinf(rl[b, h]):
                    assert np.isinf(l[b, h]) and not o[b, h].any()
                    continue
                err = np.linalg.norm(o[b, h] - r[b, h]) / np.linalg.norm(r[b, h])
                assert err <= REL_L2_TOL, (call, b, h, err)
                assert abs(l[b, h] - rl[b, h]) <= LSE_ABS_TOL, (call, b, h)


def test_noalloc_rejects_problems_beyond_its_scratch():
    import __graft_entry__
    __graft_entry__.build()
    import lsh_sampled_sparse_simhash_b200 as mp
    from lsh_sampled_sparse_simhash_b200._binding import _CShape
    big = _CShape(16, 32, 8, 128, 131200, 8, 75, 4, 64, 0)  # the ragged 16 x 128k batch
    n = ctypes.c_size_t()
    assert mp.library().mp_decode_workspace_bytes(ctypes.byref(big), 131073, ctypes.byref(n)) == 0
    assert n.value > 16 << 20
    rc = mp.library().mp_decode_attend_noalloc(ctypes.byref(big), *([16] * 6), 131073, 16, 16, 16, None, None)
    assert rc == mp.MP_ERR_TOO_LARGE
    assert "MP_ERR_TOO_LARGE" in mp.status_string(rc)

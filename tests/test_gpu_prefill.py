"""Streamed prefill hashing (mp_hash_keys_range): block-by-block hashing of a
growing cache gives the same codes as one bulk mp_hash_keys call (same kernel
and arithmetic, so bit for bit) and matches the oracle; and a range hash on a
second stream next to decodes over the tokens below the range changes
neither result."""
import numpy as np
import pytest
import torch

from gpu_harness import Run, code_mismatch, host, oracle_unit_codes
from workloads import WORKLOADS

import lsh_sampled_sparse_simhash_b200 as mp

pytestmark = pytest.mark.gpu

TINY = WORKLOADS["tiny"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("layout", ["bytes", "planes"])
@pytest.mark.parametrize("k_bits,n_tables", [(8, 75), (10, 150)])
def test_blockwise_hash_equals_bulk_hash_and_oracle(layout, k_bits, n_tables):
    if layout == "bytes" and k_bits != 8:
        pytest.skip("byte codes are K = 8 only")
    w = TINY.with_(name="pf", batch=2, n_q_heads=8, n_kv_heads=2, context=3000, k_bits=k_bits, n_tables=n_tables,
                   n_planted=8, seed=2101, code_layout=layout)
    bulk = Run(w)
    bulk.hash_keys(w.context)
    torch.cuda.synchronize()
    ref_codes = bulk.codes.clone()

    run = Run(w)
    run.codes.zero_()
    # contiguous blocks, each starting on a 128-token tile (as a chunked prefill appends them)
    blocks = [(0, 1024), (1024, 128), (1152, 1024), (2176, w.context - 2176)]
    for first, n in blocks:
        mp.hash_keys_range(run.shape, run.K, run.W, first, n, run.codes)
    torch.cuda.synchronize()
    # bit-identical to the bulk call over the hashed tokens
    for b in range(w.batch):
        for kh in range(w.n_kv_heads):
            np.testing.assert_array_equal(run.codes_logical(b, kh, w.context), bulk.codes_logical(b, kh, w.context))
    # and within the near-zero tolerance of the oracle
    for b in range(w.batch):
        for kh in range(w.n_kv_heads):
            c, m = oracle_unit_codes(run.inp, w, b, kh, w.context)
            bad, _ = code_mismatch(run.codes_logical(b, kh, w.context), c, m, w.k_bits)
            assert bad == 0
    assert torch.equal(run.codes, ref_codes)  # and nothing outside the hashed tokens differs


def test_range_hash_beside_decode_on_two_streams():
    """Decode over the first N0 tokens on one stream while the next block of
    the cache is hashed on another: both results equal the serial ones."""
    w = TINY.with_(name="pf2", batch=2, n_q_heads=8, n_kv_heads=2, context=6000, k_bits=10, n_tables=150,
                   n_planted=16, seed=2102)
    n0, first, n = 4000, 4096, 1904  # decode reads tokens < 4000; the range starts on the next tile
    run = Run(w)
    run.hash_keys(n0)
    run.lens.fill_(n0)
    run.alloc_decode(n0)
    torch.cuda.synchronize()
    serial = run.decode(member=False)
    mp.hash_keys_range(run.shape, run.K, run.W, first, n, run.codes)
    torch.cuda.synchronize()
    serial_codes = run.codes.clone()

    run.codes.copy_(serial_codes)
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    side.wait_stream(main)
    outs = []
    for _ in range(4):
        with torch.cuda.stream(side):
            mp.hash_keys_range(run.shape, run.K, run.W, first, n, run.codes, stream=side)
        mp.decode_attend(run.shape, run.q, run.W, run.codes, run.K, run.V, run.lens, run.max_len, run.out, run.lse,
                         run.ns, run.ws)
        outs.append((run.out.clone(), run.lse.clone(), run.ns.clone()))
    main.wait_stream(side)
    torch.cuda.synchronize()
    assert mp.read_status(run.ws) == 0
    for o, l, ns in outs:
        assert torch.equal(o.cpu(), torch.from_numpy(serial["out"]))
        assert torch.equal(l.cpu(), torch.from_numpy(serial["lse"]))
        assert torch.equal(ns.cpu(), torch.from_numpy(serial["ns"]))
    assert torch.equal(run.codes, serial_codes)

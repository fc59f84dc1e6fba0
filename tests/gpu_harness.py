"""GPU-side harness for the parity tests: moves seeded inputs to the device,
drives the library through its C ABI and compares against the fp64 oracle.
(Test infrastructure: imports both the library binding and the oracle.)"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np
import torch

import lsh_sampled_sparse_simhash_b200 as mp
import oracle
from layout import pack_codes, unpack_codes
from workloads import Workload, make_inputs

REL_L2_TOL = 2e-3   # per head, against the fp64 oracle on the same candidate set
LSE_ABS_TOL = 1e-3
NEAR_ZERO = 1e-4    # bits with |k.w| <= 1e-4 |k||w| may differ (fp32 vs fp64 sums)


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor, dtype=None) -> np.ndarray:
    a = t.cpu().numpy()
    if dtype is not None:
        a = a.view(dtype)
    return a


LAYOUTS = {"auto": 0, "bytes": 1, "planes": 2}


def shape_of(w: Workload) -> mp.Shape:
    return mp.Shape(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.capacity, w.k_bits, w.n_tables,
                    w.sink, w.window, LAYOUTS[w.code_layout])


class Run:
    """Device buffers of one workload and the library calls on them."""

    def __init__(self, w: Workload, inputs: Optional[dict] = None):
        self.w = w
        self.inp = inputs if inputs is not None else make_inputs(w)
        self.shape = shape_of(w)
        i = self.inp
        self.W = dev(i["W"])
        self.q = dev(i["q"])
        self.K = dev(i["K"])
        self.V = dev(i["V"])
        self.lens = dev(i["seq_lens"].astype(np.int32))
        self.k_new = dev(i["k_new"])
        self.v_new = dev(i["v_new"])
        kind, cshape = mp.codes_shape(self.shape)
        self.codes = torch.zeros(cshape, dtype=torch.uint8 if kind == "uint8" else torch.int32, device="cuda")
        self.max_len = int(i["seq_lens"].max()) if len(i["seq_lens"]) else 0
        self.alloc_decode(self.max_len)

    def alloc_decode(self, max_len: int):
        w = self.w
        self.max_len = max_len
        self.ws = torch.empty(mp.decode_workspace_bytes(self.shape, max_len), dtype=torch.uint8, device="cuda")
        self.out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
        self.lse = torch.empty((w.batch, w.n_q_heads), dtype=torch.float32, device="cuda")
        self.ns = torch.empty((w.batch, w.n_q_heads), dtype=torch.int32, device="cuda")

    # ---- library calls ----
    def hash_keys(self, n_tokens: Optional[int] = None, seq_lens=None):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        mp.hash_keys(self.shape, self.K, self.W, self.max_len if n_tokens is None else n_tokens, self.codes,
                     seq_lens=seq_lens, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, "hash kernel reported a stalled pipeline"

    def hash_queries(self) -> np.ndarray:
        qc = torch.zeros((self.w.batch, self.w.n_q_heads, self.w.n_tables), dtype=torch.int16, device="cuda")
        mp.hash_queries(self.shape, self.q, self.W, qc)
        torch.cuda.synchronize()
        return host(qc, np.uint16)

    def set_codes(self, logical: np.ndarray, units: Optional[Sequence] = None):
        """Writes oracle codes (logical [B,Hkv,N,L] or, with units, [n][N,L])."""
        w = self.w
        planes = self.shape.planes
        if units is None:
            packed = pack_codes(logical, w.k_bits, w.capacity, planes)
            self.codes.copy_(dev(packed).view(self.codes.dtype))
        else:
            for (b, kh), lg in zip(units, logical):
                packed = pack_codes(lg, w.k_bits, w.capacity, planes)
                self.codes[b, kh].copy_(dev(packed).view(self.codes.dtype))

    def codes_logical(self, b: int, kh: int, n: int) -> np.ndarray:
        a = host(self.codes[b, kh])
        if self.shape.planes:
            a = a.view(np.uint32)
        return unpack_codes(a, self.w.k_bits, self.w.n_tables, n, self.shape.planes)

    def alloc_q8(self):
        """int8 key rows (128 values + the 16-byte record), filled with a
        sentinel (0x55 bytes) so that rows the library does not write stay
        recognisable."""
        w = self.w
        self.k8 = torch.full((w.batch, w.n_kv_heads, w.capacity, mp.Q8_ROW_BYTES), 0x55, dtype=torch.int8,
                             device="cuda")

    def decode(self, qcodes_in: Optional[np.ndarray] = None, member: bool = True, path: int = 0, q8: bool = False,
               skip_scan: bool = False):
        """One decode step; with q8 the K rows come from the int8 copy."""
        w = self.w
        mem = torch.zeros((w.batch, w.n_q_heads, w.capacity), dtype=torch.uint8, device="cuda") if member else None
        qco = torch.zeros((w.batch, w.n_q_heads, w.n_tables), dtype=torch.int16, device="cuda")
        qci = dev(qcodes_in) if qcodes_in is not None else None
        if q8:
            mp.decode_attend_q8(self.shape, self.q, self.W, self.codes, self.k8, self.V, self.lens,
                                self.max_len, self.out, self.lse, self.ns, self.ws, qcodes_in=qci, qcodes_out=qco,
                                member_out=mem, path=path)
        else:
            mp.decode_attend(self.shape, self.q, self.W, self.codes, self.K, self.V, self.lens, self.max_len,
                             self.out, self.lse, self.ns, self.ws, qcodes_in=qci, qcodes_out=qco, member_out=mem,
                             path=path, skip_scan=skip_scan)
        torch.cuda.synchronize()
        res = dict(out=host(self.out), lse=host(self.lse), ns=host(self.ns), qcodes=host(qco, np.uint16))
        if member:
            res["member"] = host(mem)
        res["status"] = mp.read_status(self.ws)
        return res


# ---------------------------------------------------------------- oracle ----

def oracle_unit_codes(inp: dict, w: Workload, b: int, kh: int, n: int):
    """Oracle SimHash codes [n, L] and margins [n, L*K] of one unit's keys."""
    return oracle.simhash(inp["K"][b, kh, :n], inp["W"], w.k_bits, w.n_tables, margin=True)


def oracle_query_codes(inp: dict, w: Workload):
    return oracle.simhash(inp["q"], inp["W"], w.k_bits, w.n_tables, margin=True)


def code_mismatch(gpu: np.ndarray, ref: np.ndarray, margin: np.ndarray, K: int):
    """(bits that differ beyond the near-zero tolerance, exempt flips)."""
    diff = (gpu ^ ref).astype(np.uint32)
    bits = ((diff[..., None] >> np.arange(K, dtype=np.uint32)) & 1).astype(bool)
    bits = bits.reshape(*diff.shape[:-1], -1)
    exempt = margin <= NEAR_ZERO
    return int((bits & ~exempt).sum()), int((bits & exempt).sum())


def oracle_decode_units(inp: dict, w: Workload, units, kcodes_units, qcodes, keys: Optional[dict] = None):
    """Oracle decode of selected (b, kv head) units given codes (and, with
    `keys`, other key rows [n, d] for the units it maps: the codes stay those
    given).  Returns {(b, kh): (out [G,d], lse [G], ns [G], member [G, n])}."""
    G = w.group
    res = {}
    for (b, kh), kc in zip(units, kcodes_units):
        n = int(inp["seq_lens"][b])
        q = inp["q"][b:b + 1, kh * G:(kh + 1) * G]
        Kc = inp["K"][b:b + 1, kh:kh + 1, :n] if keys is None else keys[(b, kh)][None, None, :n]
        Vc = inp["V"][b:b + 1, kh:kh + 1, :n]
        qc = qcodes[b:b + 1, kh * G:(kh + 1) * G]
        out, lse, ns, mem = oracle.decode(q, Kc, Vc, kc[None, None, :n], qc, np.array([n], np.int32),
                                          Kbits=w.k_bits, L=w.n_tables, sink=w.sink, window=w.window,
                                          want_member=True)
        res[(b, kh)] = (out[0], lse[0], ns[0], mem[0])
    return res


def rel_l2(a: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.linalg.norm(ref))
    return float(np.linalg.norm(a - ref)) / (den if den > 0 else 1.0)


def check_outputs(gpu: dict, ref: dict, w: Workload, check_member: bool = True, rel_tol: float = REL_L2_TOL,
                  lse_tol: float = LSE_ABS_TOL):
    """Asserts member / n_sampled exact and out / lse within tolerance on every
    unit of `ref`.  Returns the worst relative L2 seen."""
    G = w.group
    worst = 0.0
    for (b, kh), (out, lse, ns, mem) in ref.items():
        n = mem.shape[-1]
        hs = slice(kh * G, (kh + 1) * G)
        if check_member:
            np.testing.assert_array_equal(gpu["member"][b, hs, :n], mem, err_msg=f"member b={b} kh={kh}")
            np.testing.assert_array_equal(gpu["ns"][b, hs], ns, err_msg=f"n_sampled b={b} kh={kh}")
        for g in range(G):
            o = gpu["out"][b, kh * G + g]
            if math.isinf(lse[g]):
                assert math.isinf(gpu["lse"][b, kh * G + g]) and not o.any()
                continue
            e = rel_l2(o.astype(np.float64), out[g])
            worst = max(worst, e)
            assert e <= rel_tol, (b, kh, g, e)
            assert abs(gpu["lse"][b, kh * G + g] - lse[g]) <= lse_tol, (b, kh, g, gpu["lse"][b, kh * G + g], lse[g])
    return worst

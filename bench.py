#!/usr/bin/env python
"""Benchmark of one LSH-sampled decode layer-step (MagicPIG hot path) on B200.

A step is one decode of every sequence of the batch:
  mp_append_token   one new token per sequence (K/V row + its SimHash codes,
                    length + 1),
  mp_decode_attend  query hash, collision scan + compaction, sampled attention
                    with the -log u correction, exact sink/window set, LSE merge,
over the post-append context.  The key-hash build of the cached keys
(mp_hash_keys, a tcgen05 tensor-core GEMM) is a prefill cost: it is timed on
its own (`breakdown.hash_*`, against the bf16 tensor peak), except for the
16k-token Llama-3.1-8B-shaped layer, whose step specification hashes every
cached key, so there the step is hash + append + decode.

Metric: decode context tokens scanned per second per layer-step: the sum over
sequences of the post-append length, divided by the step's device time;
`roofline` is the step's algorithmic HBM bytes (key codes + the unique
sampled K/V rows + the exact-set rows) over the same time, against the
measured HBM copy bandwidth.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One process per GPU (torchrun for N > 1): every rank runs an independent
replica with its own seed (no collective on the data path), so `value` is the
sum over ranks of the tokens scanned divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "ragged16"
HASH_IN_STEP = ("llama8b_16k",)  # workloads whose step hashes every cached key
FLUSH_BYTES = 256 << 20  # > 126 MB L2
METRIC = "decode context-tokens scanned/s per layer-step"
HASH_IMPL = "tcgen05-bf16"   # implementation of mp_hash_keys in this build
# The pages' own system-level claim, reported as context only (other
# hardware, other system: CPU-side sampled attention next to GPU attention).
PAGES_CLAIM = dict(
    claim="MagicPIG decoding throughput 1.76-4.99x over GPU-only attention",
    hardware="CPU + GPU: Intel CPUs with AVX512 (AVX512_BF16 for bf16) for the sampled attention; "
             "GPU model not stated",
    source="sourcepulse project page, 'Highlighted Details' and 'Quick Start & Requirements'",
    role="context, not the target")


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-overlap", action="store_true", help="skip the streamed-prefill overlap measurement")
    p.add_argument("--code-layout", default=None, choices=["auto", "bytes", "planes"],
                   help="key-code layout (default: the workload's, i.e. bytes for K=8, planes for K=10)")
    p.add_argument("--no-graph", action="store_true",
                   help="launch every timed step eagerly instead of replaying a captured CUDA graph")
    p.add_argument("--k-format", default="bf16", choices=["bf16", "int8"],
                   help="K rows gathered by the attention: the bf16 cache, or its int8 copy (per-row "
                        "power-of-two scale; opt-in reduced precision, written by mp_quantize_keys and "
                        "mp_append_token_q8)")
    p.add_argument("--decode-path", default="auto", choices=["auto", "split", "fused", "tc"],
                   help="decode kernels: auto, split (scan then attention), fused (one kernel; bit planes) or tc "
                        "(scan then the tcgen05 attention kernel)")
    args = p.parse_args(argv)
    if args.k_format == "int8" and args.decode_path in ("fused", "tc"):
        p.error("--k-format int8 runs on the split path only (--decode-path auto or split)")
    return args


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    sm_max_mhz=float(d.get("sm_max_mhz", 1965.0)), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, sm_max_mhz=1965.0, source="fallback")


def reduce_over_ranks(total_ms, tokens, device, world):
    """Whole-job numbers: the slowest rank's device time and the sum of the
    tokens every rank processed (one replica per rank)."""
    import torch
    t = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    n = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return t.item(), n.item()


def workload_for_rank(name, rank, code_layout=None):
    import workloads
    w = workloads.get(name)
    if code_layout:
        w = w.with_(code_layout=code_layout)
    return w.with_(seed=w.seed + 7919 * rank) if rank else w


def hash_in_step(w) -> bool:
    return w.name in HASH_IN_STEP


def step_tokens(lens_after):
    return int(np.sum(lens_after))


def row_bytes(w, k_format="bf16"):
    """Bytes of one gathered (token, kv head) row: k + v in bf16 (512 at
    d = 128), or the 144-byte int8 row (values and {scale, norm} record) and
    the bf16 v (400)."""
    return (w.head_dim + 16 if k_format == "int8" else 2 * w.head_dim) + 2 * w.head_dim


def decode_bytes(w, lens_after, union_rows, k_format="bf16"):
    """Algorithmic HBM bytes of one decode over post-append lengths: the key
    codes of every (token, kv head) (L*K/8 bytes each), the unique sampled
    K/V rows and the exact-set rows (row_bytes each)."""
    LK = w.n_tables * w.k_bits
    code_bytes = int(np.sum(lens_after)) * w.n_kv_heads * LK // 8
    d_rows = sum(min(w.sink, int(n)) + int(n) - max(min(w.sink, int(n)), int(n) - w.window)
                 for n in lens_after) * w.n_kv_heads
    return code_bytes + (union_rows + d_rows) * row_bytes(w, k_format), code_bytes, d_rows


def step_description(w):
    if hash_in_step(w):
        return "hash all cached keys + append 1 token/sequence + LSH-sampled decode"
    return "append 1 token/sequence + LSH-sampled decode (key-hash build timed apart)"


def code_layout_of(w):
    """The key-code layout the library uses for this workload."""
    if w.code_layout != "auto":
        return w.code_layout
    from lsh_sampled_sparse_simhash_b200 import auto_planes
    return "planes" if auto_planes(w.batch, w.n_kv_heads, w.capacity, w.k_bits) else "bytes"


def config_of(w):
    """The workload, identical on both arms (no launch or kernel-path keys)."""
    return dict(workload=w.name, batch=w.batch, q_heads=w.n_q_heads, kv_heads=w.n_kv_heads,
                head_dim=w.head_dim, context=w.context, ragged_min=w.ragged_min or None, k_bits=w.k_bits,
                n_tables=w.n_tables, sink=w.sink, window=w.window, planted_per_kv_head=w.n_planted,
                code_layout=code_layout_of(w),
                step=step_description(w),
                l2="flushed between timed steps (256 MiB write)", parallelism="replicas (1 rank = 1 GPU)")


# ------------------------------------------------------------- clocks ----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smmax=float(f[2]), reasons=[
                    n for n, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                       "sw_power_cap"), f[5:9]) if v.lower() == "active"]))
            except ValueError:
                continue
        if not rows:
            return None
        reasons = sorted({r for row in rows for r in row["reasons"]})
        return dict(sm_mhz=statistics.median(r["sm"] for r in rows), sm_max_mhz=max(r["smmax"] for r in rows),
                    reasons=reasons, samples=len(rows))


# --------------------------------------------------------- our arm ----

class Bench:
    def __init__(self, w, device, path="auto", k_format="bf16"):
        import torch
        import lsh_sampled_sparse_simhash_b200 as mp
        from workloads import make_inputs
        self.mp, self.torch, self.w = mp, torch, w
        inp = make_inputs(w)
        self.inp = inp
        self.shape = mp.Shape(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.capacity, w.k_bits,
                              w.n_tables, w.sink, w.window,
                              {"auto": mp.MP_CODES_AUTO, "bytes": mp.MP_CODES_BYTES,
                               "planes": mp.MP_CODES_PLANES}[w.code_layout])

        def dev(a):
            return torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a)).to(device)

        self.W, self.K, self.V = dev(inp["W"]), dev(inp["K"]), dev(inp["V"])
        # The per-step inputs (q, k_new, v_new, lengths) live in one device
        # buffer and the outputs (out, lse, n_sampled) in another, so that the
        # end-to-end measurement moves each direction with a single copy.
        step_in = [inp["q"].view(np.int16), inp["k_new"].view(np.int16), inp["v_new"].view(np.int16),
                   inp["seq_lens"].astype(np.int32)]
        self.in_host = _pack_host(step_in)
        self.in_dev = torch.from_numpy(self.in_host).to(device)
        self.q, self.k_new, self.v_new, self.lens = _views(self.in_dev, step_in)
        self.lens0 = self.lens.clone()
        self.prefill = int(inp["seq_lens"].max())
        self.max_len = self.prefill + 1
        kind, cshape = mp.codes_shape(self.shape)
        self.codes = torch.zeros(cshape, dtype=torch.uint8 if kind == "uint8" else torch.int32, device=device)
        self.ws = torch.empty(mp.decode_workspace_bytes(self.shape, self.max_len), dtype=torch.uint8, device=device)
        B, Hq, d = w.batch, w.n_q_heads, w.head_dim
        step_out = [np.zeros((B, Hq, d), np.float32), np.zeros((B, Hq), np.float32), np.zeros((B, Hq), np.int32)]
        self.out_dev = torch.from_numpy(_pack_host(step_out)).to(device)
        self.out, self.lse, self.ns = _views(self.out_dev, step_out)
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.tokens = step_tokens(inp["seq_lens"] + 1)
        self.path = {"auto": mp.MP_PATH_AUTO, "split": mp.MP_PATH_SPLIT, "fused": mp.MP_PATH_FUSED,
                     "tc": mp.MP_PATH_TC}[path]
        self.graph_error = None
        self.with_hash = hash_in_step(w)
        self.q8 = k_format == "int8"
        if self.q8:
            self.k8 = torch.empty((B, w.n_kv_heads, w.capacity, mp.Q8_ROW_BYTES), dtype=torch.int8, device=device)
        fused = self.path == mp.MP_PATH_FUSED
        # append 1, decode: qhash + (scan, attention | fused) + merge; hash 1
        # (and with int8 keys the quantisation, 1) if in the step
        self.launches_per_step = 1 + (3 if fused else 4) + ((2 if self.q8 else 1) if self.with_hash else 0)
        # prefill: the codes of the cached keys (the step's append adds the new token's)
        self.build()
        torch.cuda.synchronize()

    def hash(self):
        """The key-hash build of the cached keys."""
        self.mp.hash_keys(self.shape, self.K, self.W, self.prefill, self.codes, seq_lens=self.lens0)

    def quantize(self):
        """The int8 copy of the cached keys (with --k-format int8)."""
        if self.q8:
            self.mp.quantize_keys(self.shape, self.K, self.k8, n_tokens=self.prefill,
                                  seq_lens=self.lens0)

    def build(self):
        """Everything a prefill leaves in the cache: codes (and the int8 copy)."""
        self.hash()
        self.quantize()

    def append(self):
        if self.q8:
            self.mp.append_token_q8(self.shape, self.k_new, self.v_new, self.W, self.K, self.V, self.codes,
                                    self.lens, self.k8)
        else:
            self.mp.append_token(self.shape, self.k_new, self.v_new, self.W, self.K, self.V, self.codes, self.lens)

    def decode(self, member_out=None):
        if self.q8:
            self.mp.decode_attend_q8(self.shape, self.q, self.W, self.codes, self.k8, self.V,
                                     self.lens, self.max_len, self.out, self.lse, self.ns, self.ws,
                                     member_out=member_out, path=self.path)
        else:
            self.mp.decode_attend(self.shape, self.q, self.W, self.codes, self.K, self.V, self.lens, self.max_len,
                                  self.out, self.lse, self.ns, self.ws, member_out=member_out, path=self.path)

    def calls(self):
        """The library calls of one step (the lengths are reset before it)."""
        if self.with_hash:
            self.build()
        self.append()
        self.decode()

    def step(self):
        self.lens.copy_(self.lens0, non_blocking=True)
        self.calls()

    def union_rows(self):
        """Unique sampled (token, kv head) rows of one decode (for the bytes roofline)."""
        torch = self.torch
        w = self.w
        self.step()
        mem = torch.zeros((w.batch, w.n_q_heads, w.capacity), dtype=torch.uint8, device=self.q.device)
        self.decode(member_out=mem)
        torch.cuda.synchronize()
        m = mem.view(w.batch, w.n_kv_heads, w.group, w.capacity).amax(dim=2)
        u = int(m.sum().item())
        del mem, m
        return u, float(self.ns.float().mean().item())

    def warm(self, warmup):
        for _ in range(warmup):
            self.flush.zero_()
            self.step()
        self.torch.cuda.synchronize()

    def events(self, steps, n=2):
        torch = self.torch
        return [[torch.cuda.Event(enable_timing=True) for _ in range(n)] for _ in range(steps)]

    def preroll(self, seconds, graph=None):
        torch = self.torch
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            for _ in range(8):
                self.flush.zero_()
                self.lens.copy_(self.lens0, non_blocking=True)
                if graph is not None:
                    graph.replay()
                else:
                    self.calls()
            torch.cuda.synchronize()

    def capture(self):
        """Captures one step's calls (every kernel of the step, programmatic
        launch edges included) in a CUDA graph; None if capture is not
        possible here."""
        torch = self.torch
        try:
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.calls()
            torch.cuda.synchronize()
            return g
        except Exception as exc:  # report the eager fallback in the JSON line
            self.graph_error = f"{type(exc).__name__}: {exc}"
            torch.cuda.synchronize()
            return None

    def run_timed(self, ev, graph=None):
        """K steps, one event pair per step (no events between the calls, which
        would serialise the programmatic launch chain); with a graph, each step
        is one replay of the captured calls.  L2 flushed before each step."""
        for e in ev:
            self.flush.zero_()
            self.lens.copy_(self.lens0, non_blocking=True)
            e[0].record()
            if graph is not None:
                graph.replay()
            else:
                self.calls()
            e[1].record()

    def run_breakdown(self, steps):
        """Per-call device times (events around each call, L2 flushed before
        each call): the key-hash build, the append and the decode."""
        torch = self.torch
        res = {"hash": [], "append": [], "decode": []}
        for _ in range(steps):
            for name, fn in (("hash", self.hash), ("append", self.append), ("decode", self.decode)):
                if name == "append":
                    self.lens.copy_(self.lens0, non_blocking=True)
                self.flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                res[name].append((e0, e1))
        torch.cuda.synchronize()
        return {k: statistics.mean(a.elapsed_time(b) for a, b in v) for k, v in res.items()}

    def prefill_overlap(self, iters=10):
        """Streamed prefill beside decoding: a block of R tokens per unit hashed
        with mp_hash_keys_range on a side stream while mp_decode_attend runs on
        the main stream.  The block re-hashes cached tokens, which rewrites
        identical codes, so the decode's result is unaffected.  Device times
        (events on the main stream after joining the side stream)."""
        torch, mp, w = self.torch, self.mp, self.w
        R = max(128, (min(int(self.inp["seq_lens"].min()), 32768) // 128) * 128)
        side = torch.cuda.Stream()
        main = torch.cuda.current_stream()

        def hash_block(stream):
            mp.hash_keys_range(self.shape, self.K, self.W, 0, R, self.codes, stream=stream)

        def timed(fn):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            ts = []
            for _ in range(iters):
                self.flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                e1.synchronize()
                ts.append(e0.elapsed_time(e1))
            return statistics.mean(ts)

        def both():
            side.wait_stream(main)
            with torch.cuda.stream(side):
                hash_block(side)
            self.decode()
            main.wait_stream(side)

        t_dec = timed(self.decode)
        t_hash = timed(lambda: hash_block(main))
        t_both = timed(both)
        rows = R * w.batch * w.n_kv_heads
        return dict(block_tokens_per_unit=R, decode_ms=t_dec, hash_block_ms=t_hash, concurrent_ms=t_both,
                    overlap=(t_dec + t_hash) / t_both,
                    hash_rows_per_s_concurrent=rows / (t_both / 1e3))

    def run_e2e(self, steps, warmup, use_graph=True):
        """Public API with host buffers: per step, one H2D copy of the step's
        inputs (q, k_new, v_new, lengths, packed) from pinned memory, the
        step's calls, and one D2H copy of out / lse / n_sampled (packed) into
        pinned memory; device-timed.  When the step hashes the cached keys,
        the H2D copy runs on a second stream beside that hash (which does not
        read those inputs) and the append waits for both."""
        torch = self.torch
        hin = torch.from_numpy(self.in_host).pin_memory()
        hout = torch.empty(self.out_dev.shape, dtype=torch.uint8).pin_memory()
        h2d = hin.numel()
        d2h = hout.numel()
        side = torch.cuda.Stream()

        def one_step():
            main = torch.cuda.current_stream()
            if self.with_hash:
                side.wait_stream(main)
                with torch.cuda.stream(side):
                    self.in_dev.copy_(hin, non_blocking=True)
                self.build()
                main.wait_stream(side)
            else:
                self.in_dev.copy_(hin, non_blocking=True)
            self.append()
            self.decode()
            hout.copy_(self.out_dev, non_blocking=True)

        graph = None
        if use_graph:  # the copies are captured too: every replay moves the step's bytes
            try:
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    one_step()
                torch.cuda.synchronize()
            except Exception:
                graph = None
                torch.cuda.synchronize()
        times = []
        for i in range(warmup + steps):
            self.flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            if graph is not None:
                graph.replay()
            else:
                one_step()
            e.record()
            e.synchronize()
            if i >= warmup:
                times.append(s.elapsed_time(e))
        return statistics.mean(times), h2d, d2h, graph is not None


def _pack_host(arrays):
    """Concatenates arrays into one uint8 buffer, each starting on 256 bytes."""
    off, spans = 0, []
    for a in arrays:
        spans.append(off)
        off += (a.nbytes + 255) // 256 * 256
    buf = np.zeros(off, np.uint8)
    for a, o in zip(arrays, spans):
        buf[o:o + a.nbytes] = np.ascontiguousarray(a).view(np.uint8).ravel()
    return buf


def _views(buf, arrays):
    """Typed views of a packed device buffer (layout of _pack_host)."""
    import torch
    tmap = {np.dtype(np.int16): torch.int16, np.dtype(np.int32): torch.int32, np.dtype(np.float32): torch.float32}
    out, off = [], 0
    for a in arrays:
        out.append(buf[off:off + a.nbytes].view(tmap[a.dtype]).view(a.shape))
        off += (a.nbytes + 255) // 256 * 256
    return out


def traffic_record(kernel, workload, layout):
    """DRAM bytes (read + write) per call from a committed ncu capture, keyed
    kernel@workload:layout, if the kernel source it was taken on is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        recs = json.load(open(path))
    except ValueError:
        return None
    rec = recs.get(f"{kernel}@{workload}:{layout}")
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or code_fingerprint(src) != rec["code_sha256"]:
        return None
    return rec["bytes_per_launch"]


def code_fingerprint(path):
    """sha256 of a C/CUDA source with its comments removed and whitespace
    collapsed: it changes when the code changes, not when a comment does."""
    import hashlib
    text = open(path).read()
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":  # string or char literal, copied through verbatim
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    code = " ".join("".join(out).split())
    return hashlib.sha256(code.encode()).hexdigest()


# ------------------------------------------------------ oracle (CPU) ----

class OracleSample:
    """The fp64 oracle on (sequence, kv head) units of the workload, one unit
    per step, cycling over a fixed set of units.  The unit's cached-key codes are the
    prefill (computed once, untimed, like the GPU arm's key-hash build); a
    step is what the GPU step does for the unit: SimHash of the appended key
    (and, for the workload whose step hashes every cached key, of all of
    them), the query codes of the unit's heads, the collision scan and the
    estimator over the post-append context.  A unit is 1/Hkv of a sequence,
    so its tokens count (N_b + 1) / Hkv toward the metric."""

    SAMPLE_UNITS = 4

    def __init__(self, w, inp=None):
        import oracle
        from workloads import hyperplanes_of, new_token_of, queries_of, seq_lens_of
        oracle.build()
        self.oracle, self.w = oracle, w
        self.W = inp["W"] if inp is not None else hyperplanes_of(w)
        self.q = inp["q"] if inp is not None else queries_of(w)
        self.lens = inp["seq_lens"] if inp is not None else seq_lens_of(w)
        self.k_new, self.v_new = (inp["k_new"], inp["v_new"]) if inp is not None else new_token_of(w)
        self.inp = inp
        # a fixed set of units spread over the batch (and so over its length
        # mix), each prepared once and then cycled through
        n = min(self.SAMPLE_UNITS, w.batch * w.n_kv_heads)
        self.units = [((i * w.batch) // n, i % w.n_kv_heads) for i in range(n)]
        self.cache = {}

    def _unit(self, b, kh):
        if (b, kh) not in self.cache:
            from workloads import unit_keys_values
            w, n = self.w, int(self.lens[b])
            if self.inp is not None:
                Kc, Vc = self.inp["K"][b, kh, :n], self.inp["V"][b, kh, :n]
            else:
                Kc, Vc = unit_keys_values(w, self.q, b, kh, n)
            Kc = np.concatenate([Kc, self.k_new[b, kh][None]])
            Vc = np.concatenate([Vc, self.v_new[b, kh][None]])
            codes = None if hash_in_step(w) else self.oracle.simhash(Kc[:n], self.W, w.k_bits, w.n_tables)
            self.cache[(b, kh)] = (Kc, Vc, codes)
        return self.cache[(b, kh)]

    def unit_step(self, b, kh):
        """Timed part of one unit-step; returns its metric tokens."""
        o, w = self.oracle, self.w
        Kc, Vc, codes = self._unit(b, kh)
        n = Kc.shape[0]
        t0 = time.perf_counter()
        if codes is None:
            kc = o.simhash(Kc, self.W, w.k_bits, w.n_tables)
        else:
            kc = np.concatenate([codes, o.simhash(Kc[n - 1:], self.W, w.k_bits, w.n_tables)])
        G = w.group
        q = self.q[b:b + 1, kh * G:(kh + 1) * G]
        qc = o.simhash(q, self.W, w.k_bits, w.n_tables)
        o.decode(q, Kc[None, None], Vc[None, None], kc[None, None], qc, np.array([n], np.int32),
                 Kbits=w.k_bits, L=w.n_tables, sink=w.sink, window=w.window)
        return time.perf_counter() - t0, n / w.n_kv_heads

    def describe(self):
        extra = "SimHash of all its cached keys, " if hash_in_step(self.w) else \
            "SimHash of the appended key (cached-key codes precomputed, untimed), "
        lens = [int(self.lens[b]) + 1 for b, _ in self.units]
        return (f"one (sequence, kv head) unit per step, cycling over units {self.units} (lengths {lens}): "
                f"{extra}query codes, collision scan and estimator over the post-append context; a unit counts "
                f"(N_b + 1) / {self.w.n_kv_heads} tokens")


def oracle_rate(inp, w, budget_s):
    """cpu_baseline of our arm: oracle unit-steps until ~budget_s of timed
    CPU work; tokens/s over the timed parts."""
    smp = OracleSample(w, inp)
    done_tokens, busy, k = 0.0, 0.0, 0
    while busy < budget_s and k < 200:
        b, kh = smp.units[k % len(smp.units)]
        dt, tok = smp.unit_step(b, kh)
        busy += dt
        done_tokens += tok
        k += 1
    sample = f"{k} unit-steps ({smp.describe()})"
    return done_tokens / busy, dict(kind="oracle", cores=smp.oracle.num_threads(), sample=sample,
                                   seconds=round(busy, 2))


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, on the host cores,
    each step one bounded sample of the workload (one unit-step); rank 0
    only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = workload_for_rank(args.workload, 0, args.code_layout)
    smp = OracleSample(w)
    times, toks = [], []
    for i in range(args.warmup + args.steps):
        b, kh = smp.units[i % len(smp.units)]
        dt, tok = smp.unit_step(b, kh)
        if i >= args.warmup:
            times.append(dt)
            toks.append(tok)
    value = sum(toks) / sum(times)
    unit = "tokens/s"
    line = dict(impl="reference", metric=METRIC, value=value, unit=unit, n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=1e3 * statistics.mean(times), higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic", config=config_of(w),
                step_sample=smp.describe(),
                cpu_baseline=dict(value=value, unit=unit, cores=smp.oracle.num_threads(), kind="oracle",
                                  sample=smp.describe()),
                e2e=dict(value=value, unit=unit, h2d_bytes_per_step=0, d2h_bytes_per_step=0),
                context=PAGES_CLAIM)
    print(json.dumps(line, default=_jsonable), flush=True)


def _jsonable(o):
    if hasattr(o, "item"):
        return o.item()
    raise TypeError(type(o).__name__)


# --------------------------------------------------------------- main ----

def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", local if world > 1 else 0)
    import __graft_entry__
    __graft_entry__.build()
    w = workload_for_rank(args.workload, rank, args.code_layout)
    bench = Bench(w, device, args.decode_path, args.k_format)
    union, mean_ns = bench.union_rows()

    def barrier():
        if world > 1:
            dist.barrier()

    bench.warm(args.warmup)
    graph = None if args.no_graph else bench.capture()
    for _ in range(3 if graph is not None else 0):  # warm replays
        bench.flush.zero_()
        bench.lens.copy_(bench.lens0, non_blocking=True)
        graph.replay()
    ev = bench.events(args.steps)
    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    bench.preroll(0.5, graph)  # untimed steps so the sampler sees the clocks under this load
    barrier()
    torch.cuda.synchronize()
    bench.run_timed(ev, graph)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    per_call = bench.run_breakdown(args.steps)
    total_ms, all_tokens = reduce_over_ranks(sum(step_ms), bench.tokens * args.steps, device, world)
    value = all_tokens / (total_ms / 1e3)

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h, e2e_graph = bench.run_e2e(min(args.steps, 20), 3, not args.no_graph)
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=device)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e = dict(value=bench.tokens * world / (t.item() / 1e3), unit="tokens/s", h2d_bytes_per_step=h2d,
                   d2h_bytes_per_step=d2h, ms_per_step=t.item(),
                   launch="cuda-graph replay (copies included)" if e2e_graph else "eager launches")

    if rank == 0:
        peaks = load_peaks()
        layout = config_of(w)["code_layout"]
        lens_after = bench.inp["seq_lens"] + 1
        dec_bytes, code_bytes, d_rows = decode_bytes(w, lens_after, union, args.k_format)
        LK = w.n_tables * w.k_bits
        hash_rows = int(bench.inp["seq_lens"].sum()) * w.n_kv_heads
        hash_flops = 2.0 * hash_rows * w.head_dim * LK
        hash_ms, append_ms, decode_ms = per_call["hash"], per_call["append"], per_call["decode"]
        if HASH_IMPL.startswith("tcgen05"):
            hash_bound, hash_peak, hash_unit = "tensor", peaks["bf16"], "TFLOP/s"
        else:  # fp32 FMA pipe: 148 SMs x 128 lanes x 2 flop x max SM clock
            hash_bound, hash_peak, hash_unit = "alu", 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12, "TFLOP/s"
        hash_roof = dict(kernel="mp_hash_keys (tcgen05 key-hash build)", bound=hash_bound,
                         achieved=hash_flops / (hash_ms / 1e3) / 1e12, peak=hash_peak, unit=hash_unit,
                         peak_source=peaks["source"] + " bf16 burst", algorithmic=hash_flops,
                         units=f"{hash_rows} key rows x {LK} columns",
                         traffic=traffic_record("hash_keys", w.name, layout))
        hash_roof["frac"] = hash_roof["achieved"] / hash_roof["peak"]
        dec_units = f"{int(lens_after.sum())} tokens x {w.n_kv_heads} kv heads; {union} union rows; {d_rows} exact rows"
        dec_roof = dict(kernel="mp_decode_attend (qhash + scan + attend + merge)", bound="hbm",
                        achieved=dec_bytes / (decode_ms / 1e3) / 1e9, peak=peaks["hbm"], unit="GB/s",
                        algorithmic=dec_bytes, units=dec_units,
                        traffic=traffic_record("decode" if args.k_format == "bf16" else "decode_q8", w.name, layout))
        dec_roof["frac"] = dec_roof["achieved"] / dec_roof["peak"]
        dec_roof["frac_of_nominal_8tbs"] = dec_roof["achieved"] / 8000.0  # nominal HBM3e figure, for context
        ms_step = total_ms / args.steps
        if bench.with_hash:
            # the step's largest part is the hash; the HBM-bound decode is
            # reported from its own events (breakdown loop)
            roofline = {k: dec_roof[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
            roofline["kernel"] = dec_roof["kernel"] + ", timed alone"
        else:
            ach = dec_bytes / (ms_step / 1e3) / 1e9
            roofline = dict(bound="hbm", achieved=ach, peak=peaks["hbm"], unit="GB/s", frac=ach / peaks["hbm"],
                            traffic=dec_roof["traffic"],
                            kernel="decode step: mp_append_token + mp_decode_attend (qhash + scan + attend + "
                                   "merge), timed over the timed region")
        roofline["peak_source"] = peaks["source"] + " HBM copy"
        roofline["algorithmic_bytes"] = dec_bytes
        roofline["bytes"] = dict(codes=code_bytes, union_rows=union, exact_rows=d_rows,
                                 row_bytes=row_bytes(w, args.k_format))
        roofline["frac_of_nominal_8tbs"] = roofline["achieved"] / 8000.0
        line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=world, steps=args.steps,
                    warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True,
                    scaling="weak", vs_baseline=None,
                    dtype="bf16-in/fp32-acc" if args.k_format == "bf16" else
                    "bf16 q/v + int8 k (per-row power-of-two scale)/fp32-acc", data="synthetic",
                    config=config_of(w),
                    launch=dict(decode_path=args.decode_path, k_format=args.k_format,
                                mode="cuda-graph replay per step" if graph is not None else
                                "eager launches" + (f" ({bench.graph_error})" if bench.graph_error else "")),
                    roofline=roofline,
                    breakdown=dict(hash_ms=hash_ms, append_ms=append_ms, decode_ms=decode_ms,
                                   hash_in_step=bench.with_hash,
                                   hash_roofline=hash_roof, decode_roofline=dec_roof,
                                   decode_only_tokens_per_s=bench.tokens / (decode_ms / 1e3),
                                   mean_sampled_per_head=mean_ns, union_rows=union,
                                   note="per-call times: events around each call alone, L2 flushed before "
                                        "each; the step is one graph replay with the launches overlapped"),
                    gpu_launches=bench.launches_per_step * args.steps, clocks=clk, e2e=e2e,
                    context=PAGES_CLAIM)
        if not args.no_overlap:
            line["prefill_overlap"] = bench.prefill_overlap()
        if world == 1 and not args.no_cpu_baseline:
            v, info = oracle_rate(bench.inp, w, budget_s=10.0)
            line["cpu_baseline"] = dict(value=v, unit="tokens/s", **info)
        print(json.dumps(line, default=_jsonable), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

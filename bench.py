#!/usr/bin/env python
"""Benchmark of one LSH-sampled decode layer-step (MagicPIG hot path) on B200.

A step = every row of the hot path over one batch of synthetic input:
  mp_hash_keys   SimHash of every cached key (tcgen05 tensor-core GEMM with a
                 sign-packing epilogue),
  mp_append_token  one new token per sequence (K/V row + codes, length + 1),
  mp_decode_attend query hash, collision scan + compaction, sampled attention
                 with the -log u correction, exact sink/window set, LSE merge.
Metric: decode context tokens scanned per second per layer-step
(sum over sequences of the post-append length, divided by the step time).

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

DEFAULT_WORKLOAD = "llama8b_16k"
FLUSH_BYTES = 256 << 20  # > 126 MB L2
METRIC = "decode context-tokens scanned/s per layer-step"
HASH_IMPL = "tcgen05-bf16"   # implementation of mp_hash_keys in this build


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--code-layout", default=None, choices=["auto", "bytes", "planes"],
                   help="key-code layout (default: the workload's, i.e. bytes for K=8, planes for K=10)")
    p.add_argument("--no-graph", action="store_true",
                   help="launch every timed step eagerly instead of replaying a captured CUDA graph")
    p.add_argument("--decode-path", default="auto", choices=["auto", "split", "fused"],
                   help="decode kernels: auto, split (scan then attention) or fused (one kernel; bit planes)")
    return p.parse_args()


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


def step_tokens(lens_after):
    return int(np.sum(lens_after))


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
    def __init__(self, w, device, path="auto"):
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
        self.path = {"auto": mp.MP_PATH_AUTO, "split": mp.MP_PATH_SPLIT, "fused": mp.MP_PATH_FUSED}[path]
        self.graph_error = None
        fused = self.path == mp.MP_PATH_FUSED
        # hash 1, append 1, decode: qhash + (scan, attention | fused) + merge
        self.launches_per_step = 2 + (3 if fused else 4)

    def hash(self):
        self.mp.hash_keys(self.shape, self.K, self.W, self.prefill, self.codes, seq_lens=self.lens0)

    def append(self):
        self.mp.append_token(self.shape, self.k_new, self.v_new, self.W, self.K, self.V, self.codes, self.lens)

    def decode(self):
        self.mp.decode_attend(self.shape, self.q, self.W, self.codes, self.K, self.V, self.lens, self.max_len,
                              self.out, self.lse, self.ns, self.ws, path=self.path)

    def step(self):
        self.lens.copy_(self.lens0, non_blocking=True)
        self.hash()
        self.append()
        self.decode()

    def union_rows(self):
        """Unique sampled (token, kv head) rows of one decode (for the bytes roofline)."""
        torch = self.torch
        w = self.w
        self.step()
        mem = torch.zeros((w.batch, w.n_q_heads, w.capacity), dtype=torch.uint8, device=self.q.device)
        self.mp.decode_attend(self.shape, self.q, self.W, self.codes, self.K, self.V, self.lens, self.max_len,
                              self.out, self.lse, self.ns, self.ws, member_out=mem, path=self.path)
        torch.cuda.synchronize()
        m = mem.view(w.batch, w.n_kv_heads, w.group, w.capacity).amax(dim=2)
        return int(m.sum().item()), float(self.ns.float().mean().item())

    def timed(self, steps, warmup):
        torch = self.torch
        for _ in range(warmup):
            self.flush.zero_()
            self.step()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        return ev

    def preroll(self, seconds):
        torch = self.torch
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            for _ in range(8):
                self.flush.zero_()
                self.step()
            torch.cuda.synchronize()

    def capture(self):
        """Captures one step (hash, append, decode: every kernel of the step,
        programmatic launch edges included) in a CUDA graph; None if capture
        is not possible here."""
        torch = self.torch
        try:
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.hash()
                self.append()
                self.decode()
            torch.cuda.synchronize()
            return g
        except Exception as exc:  # report the eager fallback in the JSON line
            self.graph_error = f"{type(exc).__name__}: {exc}"
            torch.cuda.synchronize()
            return None

    def run_timed(self, ev, graph=None):
        """K steps, one event pair per step (no events between the calls, which
        would serialise the programmatic launch chain); with a graph, each step
        is one replay of the captured hash + append + decode."""
        for e in ev:
            self.flush.zero_()
            self.lens.copy_(self.lens0, non_blocking=True)
            e[0].record()
            if graph is not None:
                graph.replay()
            else:
                self.hash()
                self.append()
                self.decode()
            e[1].record()

    def run_breakdown(self, ev):
        """K more steps with an event between every call: per-call device time
        for the roofline of each kernel."""
        for e in ev:
            self.flush.zero_()
            self.lens.copy_(self.lens0, non_blocking=True)
            e[0].record()
            self.hash()
            e[1].record()
            self.append()
            e[2].record()
            self.decode()
            e[3].record()

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
        three calls, and one D2H copy of out / lse / n_sampled (packed) into
        pinned memory; device-timed.  The H2D copy runs on a second stream
        next to the hash of the cached keys, which does not read those inputs;
        the append waits for both."""
        torch = self.torch
        hin = torch.from_numpy(self.in_host).pin_memory()
        hout = torch.empty(self.out_dev.shape, dtype=torch.uint8).pin_memory()
        h2d = hin.numel()
        d2h = hout.numel()
        side = torch.cuda.Stream()

        def one_step():
            main = torch.cuda.current_stream()
            side.wait_stream(main)
            with torch.cuda.stream(side):
                self.in_dev.copy_(hin, non_blocking=True)
            self.hash()
            main.wait_stream(side)
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

def oracle_unit_step(inp, w, b, kh):
    """The fp64 oracle over one (b, kv head) unit of a step: SimHash of the
    unit's post-append keys, query codes of its heads, then the decode."""
    import oracle
    n = int(inp["seq_lens"][b]) + 1
    G = w.group
    Kc = inp["K"][b, kh, :n].copy()
    Kc[n - 1] = inp["k_new"][b, kh]
    Vc = inp["V"][b, kh, :n].copy()
    Vc[n - 1] = inp["v_new"][b, kh]
    kc = oracle.simhash(Kc, inp["W"], w.k_bits, w.n_tables)
    q = inp["q"][b:b + 1, kh * G:(kh + 1) * G]
    qc = oracle.simhash(q, inp["W"], w.k_bits, w.n_tables)
    oracle.decode(q, Kc[None, None], Vc[None, None], kc[None, None], qc, np.array([n], np.int32),
                  Kbits=w.k_bits, L=w.n_tables, sink=w.sink, window=w.window)
    return n


def oracle_rate(inp, w, budget_s):
    """Units of the step in (b, kv head) order until ~budget_s of CPU work;
    the rate is scaled to the whole step by token count."""
    import oracle
    units = [(b, kh) for b in range(w.batch) for kh in range(w.n_kv_heads)]
    total_unit_tokens = sum(int(inp["seq_lens"][b]) + 1 for b, _ in units)
    done_tokens, t0, k = 0, time.perf_counter(), 0
    while time.perf_counter() - t0 < budget_s:
        b, kh = units[k % len(units)]
        done_tokens += oracle_unit_step(inp, w, b, kh)
        k += 1
    dt = time.perf_counter() - t0
    est_step = dt * total_unit_tokens / done_tokens
    value = step_tokens(inp["seq_lens"] + 1) / est_step
    sample = (f"{k} (b, kv-head) unit-steps of the {len(units)} in one step ({done_tokens} unit-tokens: SimHash "
              f"of the unit's keys + collision scan + estimator), scaled to the full step by token count")
    return value, dict(kind="oracle", cores=oracle.num_threads(), sample=sample, seconds=round(dt, 2))


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from workloads import make_inputs
    oracle.build()
    w = workload_for_rank(args.workload, 0)
    inp = make_inputs(w)
    G = w.group
    units = [(b, kh) for b in range(w.batch) for kh in range(w.n_kv_heads)]
    total_unit_tokens = sum(int(inp["seq_lens"][b]) + 1 for b, _ in units)
    rates = []
    for i in range(args.warmup + args.steps):
        b, kh = units[i % len(units)]
        t0 = time.perf_counter()
        n = oracle_unit_step(inp, w, b, kh)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            rates.append(step_tokens(inp["seq_lens"] + 1) / (dt * total_unit_tokens / n))
    value = statistics.mean(rates)
    unit = "tokens/s"
    line = dict(impl="reference", metric=METRIC, value=value, unit=unit, n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=1e3 * step_tokens(inp["seq_lens"] + 1) / value,
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                config=config_of(w),
                cpu_baseline=dict(value=value, unit=unit, cores=oracle.num_threads(), kind="oracle",
                                  sample="each step: one (b, kv-head) unit (hash of its keys + collision scan "
                                         "+ estimator), scaled to the full step by token count"),
                e2e=dict(value=value, unit=unit, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line, default=_jsonable), flush=True)


def _jsonable(o):
    if hasattr(o, "item"):
        return o.item()
    raise TypeError(type(o).__name__)


def config_of(w):
    return dict(workload=w.name, batch=w.batch, q_heads=w.n_q_heads, kv_heads=w.n_kv_heads,
                head_dim=w.head_dim, context=w.context, ragged_min=w.ragged_min or None, k_bits=w.k_bits,
                n_tables=w.n_tables, sink=w.sink, window=w.window, planted_per_kv_head=w.n_planted,
                code_layout=w.code_layout if w.code_layout != "auto" else ("bytes" if w.k_bits == 8 else "planes"),
                step="hash all cached keys + append 1 token/sequence + LSH-sampled decode",
                l2="flushed between timed steps (256 MiB write)", parallelism="replicas (1 rank = 1 GPU)")


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
    bench = Bench(w, device, args.decode_path)
    union, mean_ns = bench.union_rows()

    def barrier():
        if world > 1:
            dist.barrier()

    ev = bench.timed(args.steps, args.warmup)
    graph = None if args.no_graph else bench.capture()
    for _ in range(3 if graph is not None else 0):  # warm replays
        bench.flush.zero_()
        bench.lens.copy_(bench.lens0, non_blocking=True)
        graph.replay()
    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    bench.preroll(0.5)  # untimed steps so the sampler sees the clocks under this load
    barrier()
    torch.cuda.synchronize()
    bench.run_timed(ev, graph)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    evb = bench.timed(args.steps, 0)
    bench.run_breakdown(evb)
    torch.cuda.synchronize()
    hash_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evb)
    append_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evb)
    decode_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evb)
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
        B = w.batch
        lens_after = bench.inp["seq_lens"] + 1
        LK = w.n_tables * w.k_bits
        code_bytes = int(lens_after.sum()) * w.n_kv_heads * LK // 8
        d_rows = sum(min(w.sink, n) + n - max(min(w.sink, n), n - w.window) for n in lens_after) * w.n_kv_heads
        dec_bytes = code_bytes + (union + d_rows) * 2 * w.head_dim * 2
        hash_rows = int(bench.inp["seq_lens"].sum()) * w.n_kv_heads
        hash_flops = 2.0 * hash_rows * w.head_dim * LK
        if HASH_IMPL.startswith("tcgen05"):
            hash_bound, hash_peak, hash_unit = "tensor", peaks["bf16"], "TFLOP/s"
        else:  # fp32 FMA pipe: 148 SMs x 128 lanes x 2 flop x max SM clock
            hash_bound, hash_peak, hash_unit = "alu", 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12, "TFLOP/s"
        hash_roof = dict(kernel="mp_hash_keys", bound=hash_bound, achieved=hash_flops / (hash_ms / 1e3) / 1e12,
                         peak=hash_peak, unit=hash_unit, algorithmic=hash_flops, units=f"{hash_rows} key rows",
                         traffic=traffic_record("hash_keys", w.name, config_of(w)["code_layout"]))
        hash_roof["frac"] = hash_roof["achieved"] / hash_roof["peak"]
        dec_roof = dict(kernel="mp_decode_attend", bound="hbm", achieved=dec_bytes / (decode_ms / 1e3) / 1e9,
                        peak=peaks["hbm"], unit="GB/s", algorithmic=dec_bytes,
                        units=f"{int(lens_after.sum())} tokens x {w.n_kv_heads} kv heads; {union} union rows",
                        traffic=traffic_record("decode", w.name, config_of(w)["code_layout"]))
        dec_roof["frac"] = dec_roof["achieved"] / dec_roof["peak"]
        dec_roof["frac_of_nominal_8tbs"] = dec_roof["achieved"] / 8000.0  # nominal HBM3e figure, for context
        dominant = hash_roof if hash_ms >= decode_ms else dec_roof
        roofline = {k: dominant[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
        roofline["kernel"] = dominant["kernel"]
        roofline["peak_source"] = peaks["source"]
        line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=world, steps=args.steps,
                    warmup=args.warmup, ms_per_step=total_ms / args.steps, higher_is_better=True,
                    scaling="weak", vs_baseline=None, dtype="bf16-in/fp32-acc", data="synthetic",
                    config=dict(config_of(w), decode_path=args.decode_path,
                                launch="cuda-graph replay per step" if graph is not None else
                                "eager launches" + (f" ({bench.graph_error})" if bench.graph_error else "")),
                    roofline=roofline,
                    breakdown=dict(hash_ms=hash_ms, append_ms=append_ms, decode_ms=decode_ms,
                                   hash_roofline=hash_roof, decode_roofline=dec_roof,
                                   decode_only_tokens_per_s=bench.tokens / (decode_ms / 1e3),
                                   mean_sampled_per_head=mean_ns, union_rows=union),
                    gpu_launches=bench.launches_per_step * args.steps, clocks=clk, e2e=e2e)
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

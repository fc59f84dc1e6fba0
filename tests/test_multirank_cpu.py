"""Host logic of the multi-GPU benchmark on CPU ranks (gloo, world size 2):
every rank is an independent replica with its own inputs, and the whole-job
numbers are the slowest rank's time and the sum of the ranks' tokens."""
import os
import sys

import pytest
import torch.multiprocessing as mp_

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import workloads
    w = bench.workload_for_rank("tiny", rank)
    inp = workloads.make_inputs(w)
    total_ms, tokens = bench.reduce_over_ranks(10.0 + 5.0 * rank, 1000 * (rank + 1), torch.device("cpu"), world)
    q.put((rank, w.seed, int(inp["q"].view("int16").sum()), total_ms, tokens))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_replicas_and_reduction():
    ctx = mp_.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, seed0, sum0, t0, n0), (r1, seed1, sum1, t1, n1) = res
    assert seed0 != seed1 and sum0 != sum1  # independent replicas
    assert t0 == t1 == 15.0                 # max over ranks
    assert n0 == n1 == 3000.0               # sum over ranks

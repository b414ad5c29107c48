"""bench.py's multi-rank host logic on CPU: two gloo ranks (no GPU).

Checks what the N-GPU bench line depends on: the step time is the maximum over
ranks, the processed bytes are summed over ranks (weak scaling: every rank
runs the same step), every rank passes the barriers, and under the reference
arm only rank 0 runs the oracle and prints."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    try:
        bench.barrier(dist)
        ms = 10.0 + 5.0 * rank                   # rank 1 is the slower one
        bytes_done = 1000.0 * (rank + 1)
        t = bench.max_over_ranks(dist, ms)
        b = bench.sum_over_ranks(dist, bytes_done)
        bench.barrier(dist)

        class A:
            steps, warmup = 1, 3
        # a non-zero rank of the reference arm leaves at once, without work
        ref = bench.run_reference(A, world, rank) if rank != 0 else None
        out.put((rank, t, b, ref))
    finally:
        dist.destroy_process_group()


def test_bench_rank_reductions_gloo_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(world))
    for rank, t, b, ref in res:
        assert t == pytest.approx(15.0)          # max over ranks
        assert b == pytest.approx(3000.0)        # sum over ranks
        assert ref is None

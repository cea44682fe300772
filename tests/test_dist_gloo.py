"""World-size-2 CPU (gloo) test of the multi-process plumbing the benchmark uses for N > 1:
process-group setup from the torchrun environment, barriers, the max-over-ranks timing and
the reference arm's rank-0-only rule."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist

    class A:
        pass
    args = A()
    w, r, local = bench.dist_setup(args)
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    m = bench.max_over_ranks(1.5 + rank, w)        # per-rank "times" 1.5 and 2.5
    # the reference arm: ranks other than 0 return at once, without work
    if rank != 0:
        args.steps, args.warmup, args.seed = 1, 0, 0
        bench.run_reference(args, w, r)
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((rank, m))


def test_two_rank_gloo_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 2.5), (1, 2.5)]

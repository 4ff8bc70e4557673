"""The benchmark's multi-rank logic on CPU ranks (gloo, world size 2): each rank
runs its own batch (different seed, so no data is shared and no collective is
needed on the data path), and the job time is the slowest rank's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import argparse
        import bench
        import synth
        args = argparse.Namespace(workload="tiny", batch=0, tau=None)
        base, wl = bench.rank_workload(args, rank)
        stream = synth.queries(wl, 4)
        t = bench.max_over_ranks(1.0 + 2.0 * rank, world, "cpu")
        dist.barrier()
        q.put((rank, wl.seed, float(stream.q[1].sum()), t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_distinct_batches_and_max_time():
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    (r0, s0, x0, t0), (r1, s1, x1, t1) = res
    assert s0 != s1 and x0 != x1          # independent problems per rank
    assert t0 == t1 == 3.0                # both ranks see the slowest rank's time

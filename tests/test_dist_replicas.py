"""Host logic of the multi-GPU bench (replicas, no data-path collective) on
world-size-2 gloo process groups on CPU: per-rank seeds differ, the time
reduction is a max over ranks, the work reduction a sum."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import dfssm_synth as synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(10.0 + rank, dist)
        s = bench.sum_over_ranks(1.5, dist)
        seed = bench.replica_seed(rank)
        x = synth.activations(seed, 2, 0, 1, 256)
        q.put((rank, t, s, seed, int(x.astype("int64").sum())))
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [11.0, 11.0]          # max over ranks
    assert [r[2] for r in res] == [3.0, 3.0]            # sum over ranks
    assert res[0][3] != res[1][3]                       # each replica its own seed
    assert res[0][4] != res[1][4]                       # and its own inputs


def test_single_process_reductions_are_identity():
    import bench
    assert bench.max_over_ranks(2.5, None) == 2.5
    assert bench.sum_over_ranks(2.5, None) == 2.5


def test_work_accounting_matches_the_pages_layout():
    import bench
    import dfssm_synth as synth
    shapes = synth.stack_shapes()
    assert bench.stack_bytes(shapes, 1) == 173_420_544
    ops = bench.stack_ops(shapes, 2048)
    assert abs(ops / 1e12 - 5.129) < 0.001

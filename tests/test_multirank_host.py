"""World-size-2 checks of bench.py's multi-rank host logic on CPU (gloo):
the step time is the max over ranks and the throughput counts every rank's
tokens.  No GPU and no CUDA call."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    got = bench.max_over_ranks(ms, world, "cpu")
    out[rank] = (got, bench.tokens_per_s(8192, world, got))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_world2():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    for r in range(world):
        got, tps = res[r]
        assert got == 15.0                              # max over ranks, on every rank
        assert tps == pytest.approx(8192 * 2 / 0.015)   # all ranks' tokens / slowest time


def _vocab_worker(rank, world, port, out):
    import datetime
    import sys
    import numpy as np
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from linear_cross_entropy_cce_b200 import synthetic as syn
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    wl = syn.WORKLOADS["composite_two_segment"]
    segs = [(b, e, np.arange(e - b)[:, None]) for b, e in wl.segs()]  # row ids stand in for E
    plan = bench.vocab_shard_plan(segs, wl.V, world, rank)
    live = sum(e - b for b, e, _ in plan)
    t = torch.tensor([float(live)])
    dist.all_reduce(t)  # every rank's share adds up to the live vocabulary
    ms = 10.0 + 2.0 * rank
    out[rank] = ([(b, e, int(E[0, 0]), int(E[-1, 0]), E.shape[0]) for b, e, E in plan],
                 float(t.item()), bench.max_over_ranks(ms, world, "cpu"))
    dist.barrier()
    dist.destroy_process_group()


def test_vocab_parallel_shard_plan_world2():
    """--parallel vocab: the two ranks' shards of the composite head cover its
    live ids exactly once (the dead gap in neither), rows sliced from the
    right offsets; the step time is the max over ranks."""
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_vocab_worker, args=(world, port, out), nprocs=world,
                           start_method="spawn")
        res = dict(out)
    from linear_cross_entropy_cce_b200 import synthetic as syn
    wl = syn.WORKLOADS["composite_two_segment"]
    ids = []
    for r in range(world):
        plan, total, ms = res[r]
        assert total == wl.v_live and ms == 12.0
        for b, e, first, last, rows in plan:
            seg_b = [sb for sb, se in wl.segs() if sb <= b < se][0]
            assert first == b - seg_b and last == e - 1 - seg_b and rows == e - b
            ids.extend(range(b, e))
    live = [i for b, e in wl.segs() for i in range(b, e)]
    assert sorted(ids) == live


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5

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


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5

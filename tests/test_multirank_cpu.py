"""Host logic of the multi-GPU bench on CPU: two gloo ranks, max-over-ranks timing, weak-scaling
value, per-rank seeds (independent shards, no data-path collective)."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import sys

        sys.argv = ["bench.py", "--workload", "tiny_prefill_1k"]
        import bench

        a = bench._args()
        w = bench.workload(a, rank)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        m = bench.max_over_ranks(ms)
        out[rank] = (w.seed, m, bench.job_value(w.batch * w.n_q, world, m))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    seeds = sorted(v[0] for v in out.values())
    assert seeds == [0, 1]                       # independent shards
    assert all(v[1] == 15.0 for v in out.values())  # the job takes the slowest rank's time
    assert all(v[2] == pytest.approx(1024 * 2 / 15e-3) for v in out.values())


def test_single_process_passthrough():
    import bench

    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_value(100, 1, 10.0) == pytest.approx(1e4)

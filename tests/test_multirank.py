"""World-size-2 checks of the replica plumbing of bench.py on CPU (gloo).

The hot path has no exchange step: with N GPUs bench.py runs N independent
replicas, barriers around the timed region, takes the maximum step time over
ranks and reports the aggregate throughput.  These tests run that plumbing
with two gloo ranks, without a GPU."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    import torch.distributed as dist
    w, r, local = bench.init_ranks("gloo", timeout_s=60)
    dev = torch.device("cpu")
    bench.barrier(dev)
    step_ms = 10.0 + 5.0 * r                     # rank 1 is the slower replica
    mx = bench.reduce_over_ranks(step_ms, "max", dev)
    sm = bench.reduce_over_ranks(float(r + 1), "sum", dev)
    bench.barrier(dev)
    out[r] = (w, r, local, mx, sm, bench.aggregate_value(2.0e12, mx, w))
    dist.destroy_process_group()


def test_two_replicas_reduce_and_aggregate():
    world, port = 2, _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        w, rank, local, mx, sm, value = out[r]
        assert (w, rank, local) == (world, r, r)
        assert mx == 15.0 and sm == 3.0
        # whole-job throughput: both replicas' work over the slowest replica's time
        assert value == pytest.approx(2 * 2.0e12 / 15e-3 / 1e12)


def test_single_rank_is_identity(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    assert bench.dist_env() == (1, 0, 0)
    assert bench.reduce_over_ranks(3.5, "max", torch.device("cpu")) == 3.5
    assert bench.aggregate_value(1.0e12, 1.0, 1) == pytest.approx(1.0e3)

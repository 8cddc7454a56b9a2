"""The multi-process timing path of bench.py (replicas, one per GPU) on CPU:
two gloo ranks, each with its own device time; the reported time is the
maximum over ranks and the throughput counts every replica's work."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        out[rank] = bench.max_over_ranks(times[rank], torch.device("cpu"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    times = [12.5, 17.25]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(2, _free_port(), times, out), nprocs=2, join=True)
        assert out[0] == out[1] == max(times)


def test_single_process_and_aggregate():
    import bench
    assert bench.max_over_ranks(3.0, torch.device("cpu")) == 3.0   # no process group
    # 2 replicas of 1e12 ops in 10 ms: 200 TOPS for the whole job
    assert bench.aggregate_tops(2, 1e12, 10.0) == pytest.approx(200.0)
    assert bench.aggregate_tops(1, 1.1705e14, 64.48) == pytest.approx(1815.3, rel=1e-3)

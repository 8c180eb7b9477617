"""The N > 1 replica path of bench.py on CPU: two gloo ranks, each timing its
own replica; the job time is the max over ranks and the throughput counts
every rank's calls (weak scaling, no collective on the data path)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 3.0 - rank]  # rank 1 slower on the first timing
        dist.barrier()
        got = bench.max_over_ranks(mine)
        results[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(2, port, results), nprocs=2, join=True)
        assert results[0] == results[1] == [11.0, 3.0]


def test_job_throughput_weak_scaling():
    one = bench.job_throughput(1e12, 100, 1000.0, 1)
    two = bench.job_throughput(1e12, 100, 1000.0, 2)
    assert one == pytest.approx(100.0) and two == pytest.approx(200.0)
    # the slowest rank sets the time
    assert bench.job_throughput(1e12, 100, 2000.0, 2) == pytest.approx(100.0)


def test_gpus_flag_must_match_world_size(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr("sys.argv", ["bench.py", "--gpus", "2"])
    with pytest.raises(SystemExit):
        bench.main()

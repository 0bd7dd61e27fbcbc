"""The multi-rank timing path of bench.py on CPU with 2 gloo ranks: each rank
runs an independent replica, the job's time is the slowest rank's, and the
reported per-step value divides by all steps of all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    import bench
    mine = 10.0 + 5.0 * rank                      # per-rank elapsed ms
    got = bench.reduce_max(mine, world, torch.device("cpu"))
    v = bench.whole_job_us_per_step(got, steps=100, world=world)
    q.put((rank, got, v))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, got, v in res:
        assert got == 15.0                          # max over ranks
        assert v == pytest.approx(15.0 * 1e3 / (100 * 2))


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max(3.5, 1, None) == 3.5
    assert bench.whole_job_us_per_step(3.5, 7, 1) == pytest.approx(3500 / 7)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun the reference arm runs and prints on rank 0 alone; the
    other ranks return 0 without work or output."""
    import argparse

    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(config="tiny", batch=0, selector="quest", key_bits=4, steps=1,
                              warmup=0, gpus=2)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""

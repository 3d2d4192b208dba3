"""Host logic of the N-GPU bench path, run as two gloo ranks on the CPU.

bench.py runs one replica of the workload per GPU (independent sequences: no data-path
collective) and reports the whole job's rate over the slowest rank's device time.
"""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, local = bench.dist_setup(world)
        assert (w, r, local) == (world, rank, rank)
        ms = 10.0 * (rank + 1)             # rank 1 is the slow one
        job_ms = bench.max_over_ranks(ms, w, torch.device("cpu"))
        out[rank] = (job_ms, bench.job_rate(w, 4096, job_ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_takes_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for pr in procs:
            pr.start()
        for pr in procs:
            pr.join(120)
        assert all(pr.exitcode == 0 for pr in procs), [pr.exitcode for pr in procs]
        res = dict(out)
    for r in range(world):
        job_ms, rate = res[r]
        assert job_ms == 20.0                       # max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 4096 / 0.020)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, 1, torch.device("cpu")) == 7.5
    assert bench.job_rate(1, 1000, 500.0) == pytest.approx(2000.0)


def test_world_size_must_match_gpus(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.dist_setup(1)

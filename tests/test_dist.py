"""The bench's multi-process path (replicas, one process per GPU) on the CPU: two gloo
ranks set up the process group the way bench.py does under torchrun, take the max of
their step times over ranks and aggregate the whole-job rate; the reference arm runs on
rank 0 only."""
import argparse
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local, pg = bench.dist_setup(argparse.Namespace(impl="reference"))   # gloo backend
    assert (w, r, local) == (world, rank, rank)
    ms = bench.max_over_ranks(pg, 2.0 + rank)          # rank 1 is the slow one
    rate = bench.replica_rate(w, 5e8, ms)               # 0.5 GB per replica per step
    pg.barrier()
    pg.destroy_process_group()
    out[rank] = (ms, rate)


def test_two_gloo_ranks_take_the_max_time_and_sum_the_work():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms, rate = out[rank]
        assert ms == 3.0                                  # max over ranks
        assert rate == pytest.approx(2 * 5e8 / 3e-3)      # all ranks' bytes over the slowest time


def test_reference_arm_runs_on_rank_0_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload=2, steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args) == 0                 # returns at once, no oracle work, no output

"""Replica logic of bench.py on two CPU processes (gloo): the layer does not shard, so N GPUs run
N independent replicas; the job's time is the slowest rank's and its throughput counts every
rank's tokens.  No GPU: the timed durations are stand-ins passed by each rank."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import bench
    import synthetic as syn
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [10.0, 12.5][rank]
        slow = bench.slowest_rank_ms(my_ms, dist, torch.device("cpu"))
        cfg = syn.CONFIGS["tiny"]
        x = bench.make_batches(cfg, 2, 2, 0, bench.replica_token_base(rank), torch.device("cpu"))
        first = x[0][0, :8].tolist()
        gathered = [None] * world
        dist.all_gather_object(gathered, first)
        out[rank] = (slow, bench.job_tokens_per_s(world, 100, 1, slow), gathered)
    finally:
        dist.destroy_process_group()


def test_two_replicas_time_and_streams():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    for r in range(world):
        slow, tps, gathered = res[r]
        assert slow == 12.5                                   # max over ranks, on every rank
        assert tps == pytest.approx(2 * 100 * 1 / 12.5e-3)    # every rank's tokens / slowest time
        assert gathered[0] != gathered[1]                     # each replica has its own tokens

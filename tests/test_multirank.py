"""The multi-process (one rank per GPU) logic of bench.py, run as two gloo ranks on CPU.

Ranks time their own steps; the job's time is the slowest rank's, and the job's throughput
counts every rank's tokens.  Each rank attends over a different synthetic sequence.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    import bench
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [12.5, 30.0, 7.0, 19.0][rank]
        slowest = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        rate = bench.aggregate_rate(1000.0, world, slowest)
        # each rank's first layer: a few key values of its own synthetic sequence
        w = synth.workload("llama7b_layer_32k", Hq=2, Hkv=2)
        key = bench.rank_layer_key(0, rank)
        idx = (np.zeros((1, 1, 1, 1), dtype=np.int64), np.arange(4)[None, :, None, None],
               np.zeros((1, 1, 1, 1), dtype=np.int64), np.arange(8)[None, None, None, :])
        sample = synth.gen_k(w, key, *idx).view(np.uint16).ravel().tolist()
        out.put((rank, slowest, rate, key, sample))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ranks_agree_on_slowest_time_and_aggregate_rate(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res.sort()
    local = [12.5, 30.0, 7.0, 19.0][:world]
    for rank, slowest, rate, key, _ in res:
        assert slowest == max(local)                      # max over ranks, on every rank
        assert rate == pytest.approx(1000.0 * world / (max(local) / 1e3))
    keys = [r[3] for r in res]
    assert len(set(keys)) == world                        # a different sequence per rank
    samples = [tuple(r[4]) for r in res]
    assert len(set(samples)) == world


def test_reference_arm_runs_on_rank_zero_only():
    import bench

    class A:
        workload = "tiny_single_head"
        steps = 1
        warmup = 1

    assert bench.run_reference(A(), rank=1, world=2) == 0  # returns at once, no work

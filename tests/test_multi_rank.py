"""Multi-rank host logic of bench.py on CPU: two gloo ranks, no GPU.

Every rank runs its own independent layer (weak scaling); the only
collective is the max over ranks of the timed region.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from future_attention_targets_b200.workloads import make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + rank)                 # per-rank step time
        d = make_inputs("tiny", seed=bench.rank_seed(rank))
        out[rank] = (got, int(d["q_bits"][:64].astype(np.int64).sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()   # no fork of this (threaded) process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 2.5                  # both ranks see the slowest
    assert out[0][1] != out[1][1]                         # independent inputs per rank


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_weak_throughput():
    # 2 ranks x 2.165e12 flops in 2.5 ms (the slowest rank) = 1732 TFLOP/s for the job
    assert bench.weak_throughput(2.165e12, 2, 2.5) == pytest.approx(1732.0)
    assert bench.weak_throughput(2.165e12, 1, 2.5) == pytest.approx(866.0)

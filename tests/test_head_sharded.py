"""Head-sharded targets on CPU: two gloo ranks, the oracle as each rank's local compute.

Each rank takes its block of KV heads (with their query heads), computes the
targets of that block alone, and one all-gather assembles [H_kv, T].  The
gathered targets and the keep mask taken from them must equal the
unsharded computation on every rank.  A wrong head grouping (query heads not
following their KV head) or a gather in the wrong order fails here.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from future_attention_targets_b200.sharded import gather_targets, head_range, shard_heads
from future_attention_targets_b200.workloads import random_qk
from oracle import kvpop_oracle as oracle

T_SEQS = (170, 130)
H_Q, H_KV, D, W, S = 8, 4, 32, 16, 4
BUDGETS = (60, 50)


def _inputs():
    cu = np.concatenate([[0], np.cumsum(T_SEQS)]).astype(np.int32)
    q, k = random_qk(int(cu[-1]), H_Q, H_KV, D, seed=77)
    return q, k, cu, 1.0 / np.sqrt(D)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, cu, scale = _inputs()
        ql, kl = shard_heads(q, k, H_KV, world, rank)
        local = torch.from_numpy(oracle.future_target(ql, kl, cu, W, scale))
        full = torch.empty((H_KV, int(cu[-1])), dtype=local.dtype)
        gather_targets(local, full)
        keep = oracle.keep_mask(full.numpy(), cu, W, S, BUDGETS)
        out[rank] = (full.numpy().copy(), keep)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_unsharded():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()   # no fork of this (threaded) process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    q, k, cu, scale = _inputs()
    ref = oracle.future_target(q, k, cu, W, scale)
    ref_keep = oracle.keep_mask(ref, cu, W, S, BUDGETS)
    for r in range(world):
        tgt, keep = out[r]
        np.testing.assert_allclose(tgt, ref, rtol=1e-12, atol=0)
        assert np.array_equal(keep, ref_keep)
    assert np.array_equal(out[0][0], out[1][0])


def test_head_range_blocks():
    assert [head_range(8, 4, r) for r in range(4)] == [(0, 2), (2, 4), (4, 6), (6, 8)]
    assert head_range(8, 1, 0) == (0, 8)
    with pytest.raises(ValueError):
        head_range(8, 3, 0)          # uneven shards
    with pytest.raises(ValueError):
        head_range(8, 2, 2)          # rank outside the world


def test_shard_heads_keeps_query_groups():
    q, k, cu, _ = _inputs()
    G = H_Q // H_KV
    for r in range(2):
        ql, kl = shard_heads(q, k, H_KV, 2, r)
        h0, h1 = head_range(H_KV, 2, r)
        assert ql.flags.c_contiguous and kl.flags.c_contiguous
        assert np.array_equal(kl, k[:, h0:h1])
        assert np.array_equal(ql, q[:, h0 * G:h1 * G])
    tq, tk = shard_heads(torch.from_numpy(q.view(np.int16)), torch.from_numpy(k.view(np.int16)), H_KV, 2, 1)
    assert tq.is_contiguous() and tuple(tq.shape) == (q.shape[0], H_Q // 2, D)

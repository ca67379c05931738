"""Head-sharded targets on the GPU, through the C ABI, against the fp64 oracle.

Each KV head's targets depend only on that head and its query heads (the
scorer and the cache budget are per KV head: Qwen3-8B-KVpop-4x model card,
introduction; the aiweekly article "KVpop shrinks Qwen3 KV cache 88%",
second paragraph), so computing the heads in P separate blocks must give
every key's target within the oracle tolerance, and, since the kernels
accumulate every (head, key tile) in a fixed order whatever else is in the
launch, the unsharded result bit for bit.  The P-rank case is emulated with
P launches on one GPU, each running exactly what a rank runs (row
logsumexp, then the transposed pass with one item per (key tile, query
head) when G > 1); the collective itself runs in a one-rank NCCL group
through HeadShardedTargets.  Oracle results at full size come from
tests/oracle_cache.py.
"""
import socket

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import (check_status, future_target, future_target_split, future_targets,
                                           keep_mask, row_lse)
from future_attention_targets_b200.sharded import HeadShardedTargets, shard_heads
from future_attention_targets_b200.workloads import make_inputs
from oracle_cache import oracle_full

pytestmark = pytest.mark.gpu

TARGET_TOL = 2e-3


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def rel_err(gpu, ref):
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-3)))


def _full(d):
    q, k = dev(d["q_bits"]), dev(d["k_bits"])
    _, tgt, keep = future_targets(q, k, d["cu_seqlens"], d["window"], d["sinks"], d["budgets"], scale=d["scale"])
    return q, k, tgt, keep


def _against_oracle(name, d, tgt, keep):
    ref = oracle_full(name, d)["target"]
    tgt = tgt.cpu().numpy()
    assert rel_err(tgt, ref) <= TARGET_TOL
    np.testing.assert_array_equal(keep.cpu().numpy(),
                                  oracle.keep_mask(tgt, d["cu_seqlens"], d["window"], d["sinks"], d["budgets"]))


@pytest.mark.parametrize("name,world", [("qwen3_4b_4k", 2), ("qwen3_4b_4k", 8), ("varlen_8x", 4)])
def test_head_blocks_against_oracle(name, world):
    d = make_inputs(name)
    w = d["workload"]
    cu, W, S, scale = d["cu_seqlens"], d["window"], d["sinks"], d["scale"]
    q, k, tgt_full, keep_full = _full(d)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    parts = []
    for r in range(world):
        ql, kl = shard_heads(q, k, w.n_kv_heads, world, r)
        lse = row_lse(ql, kl, cu, scale, status=st)
        pass2 = future_target_split if w.group > 1 else future_target
        parts.append(pass2(ql, kl, cu, W, lse, scale, status=st))
    torch.cuda.synchronize()
    check_status(st)
    tgt = torch.cat(parts, 0)
    keep = keep_mask(tgt, cu, W, S, d["budgets"])
    _against_oracle(name, d, tgt, keep)
    assert torch.equal(tgt, tgt_full)
    assert torch.equal(keep, keep_full)


@pytest.mark.parametrize("name", ["qwen3_4b_4k", "varlen_8x"])
def test_one_rank_nccl_group_against_oracle(name):
    import torch.distributed as dist
    d = make_inputs(name)
    w = d["workload"]
    q, k, tgt_full, keep_full = _full(d)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        sharded = HeadShardedTargets(d["cu_seqlens"], w.n_q_heads, w.n_kv_heads, w.head_dim, d["window"],
                                     d["sinks"], d["budgets"], scale=d["scale"])
        for _ in range(2):                     # buffers are reused across calls
            tgt, keep = sharded(q, k)
        torch.cuda.synchronize()
        check_status(sharded.status)
        _against_oracle(name, d, tgt, keep)
        assert torch.equal(tgt, tgt_full)
        assert torch.equal(keep, keep_full)
    finally:
        dist.destroy_process_group()

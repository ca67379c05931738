"""Head-sharded targets on the GPU, through the C ABI.

Each KV head's targets depend only on that head and its query heads, and the
kernels accumulate every (head, key tile) in a fixed order whatever else is
in the launch, so computing the heads in P separate blocks must reproduce the
unsharded result bit for bit.  The P-rank case is emulated here with P
launches on one GPU (no collective is involved); the collective itself runs
in a one-rank NCCL group through HeadShardedTargets.
"""
import socket

import numpy as np
import pytest
import torch

from future_attention_targets_b200 import check_status, future_target, future_targets, keep_mask, row_lse
from future_attention_targets_b200.sharded import HeadShardedTargets, shard_heads
from future_attention_targets_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _full(d):
    q, k = dev(d["q_bits"]), dev(d["k_bits"])
    _, tgt, keep = future_targets(q, k, d["cu_seqlens"], d["window"], d["sinks"], d["budgets"], scale=d["scale"])
    return q, k, tgt, keep


@pytest.mark.parametrize("name,world", [("qwen3_4b_4k", 2), ("qwen3_4b_4k", 8), ("varlen_8x", 4)])
def test_head_blocks_reproduce_unsharded(name, world):
    d = make_inputs(name)
    w = d["workload"]
    cu, W, S, scale = d["cu_seqlens"], d["window"], d["sinks"], d["scale"]
    q, k, tgt_full, keep_full = _full(d)
    parts = []
    for r in range(world):
        ql, kl = shard_heads(q, k, w.n_kv_heads, world, r)
        lse = row_lse(ql, kl, cu, scale)
        parts.append(future_target(ql, kl, cu, W, lse, scale))
    tgt = torch.cat(parts, 0)
    assert torch.equal(tgt, tgt_full)
    assert torch.equal(keep_mask(tgt, cu, W, S, d["budgets"]), keep_full)


def test_one_rank_nccl_group():
    import torch.distributed as dist
    d = make_inputs("qwen3_4b_4k")
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
        assert torch.equal(tgt, tgt_full)
        assert torch.equal(keep, keep_full)
    finally:
        dist.destroy_process_group()

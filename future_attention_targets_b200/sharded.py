"""Head-sharded targets across the ranks of a process group.

Every (sequence, KV head) pair is an independent problem: the target of KV
head h needs only K head h and its G query heads, because a key's target is
the attention mass that later queries of its own group give it, and the cache
budget is kept per KV head (aiweekly article "KVpop shrinks Qwen3 KV cache
88%", second paragraph; Qwen3-8B-KVpop-4x model card, introduction).  Under
tensor-parallel attention each rank already holds a contiguous block of KV
heads with their query heads, so each rank runs the two attention passes on
its own block.  One all-gather then gives
every rank the full [H_kv, T] target, and the keep mask runs on every rank
on the gathered target, so the result is the same everywhere.

The collective is the only exchange: torch.distributed's all_gather_into_tensor
(NCCL over NVLink on GPUs, gloo on CPU).  Rank r owns KV heads
[r * H_kv / P, (r + 1) * H_kv / P), which makes the gathered rows land in
head order with no unpacking.
"""
from __future__ import annotations

import math

import numpy as np

from ._binding import (future_target, future_target_split, keep_mask, row_lse, target_split_workspace_bytes,
                       target_workspace_bytes)


def head_range(n_kv_heads: int, world: int, rank: int) -> tuple[int, int]:
    """KV heads [h0, h1) of `rank` when n_kv_heads are split evenly over `world` ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} is outside a world of {world}")
    if n_kv_heads % world != 0:
        raise ValueError(f"{n_kv_heads} KV heads do not split evenly over {world} ranks "
                         "(one all-gather needs equal shards)")
    per = n_kv_heads // world
    return rank * per, (rank + 1) * per


def shard_heads(q, k, n_kv_heads: int, world: int, rank: int):
    """This rank's contiguous copies of Q [T, H_q, d] and K [T, H_kv, d] (numpy arrays or torch tensors)."""
    h0, h1 = head_range(n_kv_heads, world, rank)
    G = q.shape[1] // n_kv_heads
    qs, ks = q[:, h0 * G:h1 * G], k[:, h0:h1]
    if isinstance(q, np.ndarray):
        return np.ascontiguousarray(qs), np.ascontiguousarray(ks)
    return qs.contiguous(), ks.contiguous()


def gather_targets(target_local, out, group=None) -> None:
    """All-gather the ranks' [H_kv / P, T] target blocks into out [H_kv, T], in head order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if out.shape[0] != world * target_local.shape[0] or out.shape[1:] != target_local.shape[1:]:
        raise ValueError(f"out {tuple(out.shape)} does not hold {world} blocks of {tuple(target_local.shape)}")
    if not (out.is_contiguous() and target_local.is_contiguous()):
        raise ValueError("gather_targets needs contiguous tensors")
    dist.all_gather_into_tensor(out, target_local, group=group)


class HeadShardedTargets:
    """row_lse + the transposed pass on this rank's KV heads, one all-gather, keep mask on all heads.

    Construct once per problem shape (buffers are allocated here, not per
    call); call with this rank's Q [T, H_q / P, d] and K [T, H_kv / P, d] on
    its GPU.  Returns (target [H_kv, T] fp32, keep [H_kv, T] uint8), identical
    on every rank.
    """

    def __init__(self, cu_seqlens, n_q_heads: int, n_kv_heads: int, head_dim: int, window: int, sinks: int,
                 budgets, scale: float | None = None, group=None, device=None):
        import torch
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.h0, self.h1 = head_range(n_kv_heads, self.world, self.rank)
        if n_q_heads % n_kv_heads != 0:
            raise ValueError("n_q_heads must be a multiple of n_kv_heads")
        self.G = n_q_heads // n_kv_heads
        self.n_local = self.h1 - self.h0
        self.cu_seqlens = np.asarray(cu_seqlens, dtype=np.int32)
        self.window, self.sinks = int(window), int(sinks)
        self.budgets = np.asarray(budgets, dtype=np.int32)
        self.scale = 1.0 / math.sqrt(head_dim) if scale is None else float(scale)
        self.head_dim = head_dim
        T = int(self.cu_seqlens[-1])
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.lse = torch.empty((self.n_local * self.G, T), dtype=torch.float32, device=dev)
        self.target_local = torch.empty((self.n_local, T), dtype=torch.float32, device=dev)
        self.target = torch.empty((n_kv_heads, T), dtype=torch.float32, device=dev)
        self.keep = torch.empty((n_kv_heads, T), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        # A shard holds few KV heads: its transposed pass takes one item per
        # (key tile, query head), whose workspace also holds partial sums.
        if self.G > 1:
            n = target_split_workspace_bytes(T, self.n_local * self.G, self.n_local, head_dim)
        else:
            n = target_workspace_bytes(T, self.n_local, self.n_local, head_dim)
        self.ws = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)

    def __call__(self, q_local, k_local, stream=None):
        import torch
        if q_local.shape[1] != self.n_local * self.G or k_local.shape[1] != self.n_local:
            raise ValueError(f"rank {self.rank} expects {self.n_local * self.G} query heads and {self.n_local} "
                             f"KV heads, got {q_local.shape[1]} and {k_local.shape[1]}")
        stream = torch.cuda.current_stream(self.target.device) if stream is None else stream
        with torch.cuda.stream(stream):
            row_lse(q_local, k_local, self.cu_seqlens, self.scale, out=self.lse, status=self.status, stream=stream)
            if self.G > 1:
                future_target_split(q_local, k_local, self.cu_seqlens, self.window, self.lse, self.scale,
                                    out=self.target_local, workspace=self.ws, status=self.status, stream=stream)
            else:
                future_target(q_local, k_local, self.cu_seqlens, self.window, self.lse, self.scale,
                              out=self.target_local, workspace=self.ws, status=self.status, stream=stream)
            gather_targets(self.target_local, self.target, self.group)
            keep_mask(self.target, self.cu_seqlens, self.window, self.sinks, self.budgets, out=self.keep,
                      stream=stream)
        return self.target, self.keep

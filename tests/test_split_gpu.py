"""The transposed pass with one work item per (key tile, query head)
(kvpop_future_target_split) against the pass with one item per (key tile,
KV head), through the C ABI.

Both sum each query head's tiles on their own and add the heads, then the
softmax column groups, in the same order, so the targets must be bit-identical;
the split pass exists so that calls with few KV heads (a group of heads, a
tensor-parallel shard) still give every SM work.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import check_status, future_target, future_target_split, row_lse
from future_attention_targets_b200.workloads import make_inputs, random_qk

pytestmark = pytest.mark.gpu


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def both(q_bits, k_bits, cu, W, scale):
    q, k = dev(q_bits), dev(k_bits)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse = row_lse(q, k, cu, scale, status=st)
    plain = future_target(q, k, cu, W, lse, scale, status=st)
    split = future_target_split(q, k, cu, W, lse, scale, status=st)
    torch.cuda.synchronize()
    check_status(st)
    return plain, split


@pytest.mark.parametrize("name", ["tiny", "qwen3_4b_4k", "varlen_8x"])
def test_split_is_bit_identical_on_workloads(name):
    """Every key of the split pass against the fp64 oracle, and bit for bit against the plain pass."""
    from oracle_cache import oracle_full
    d = make_inputs(name)
    plain, split = both(d["q_bits"], d["k_bits"], d["cu_seqlens"], d["window"], d["scale"])
    ref = oracle_full(name, d)["target"]
    got = split.cpu().numpy().astype(np.float64)
    assert float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-3))) <= 2e-3
    assert torch.equal(plain, split)


@pytest.mark.parametrize("seqlens,hq,hkv,d,W", [
    ((300,), 2, 2, 64, 16),                  # G = 1: the plain pass
    ((1, 0, 129, 257, 700), 8, 1, 128, 5),   # G = 8, one KV head, ragged tiles and an empty sequence
    ((2048,), 16, 1, 64, 0),                 # G = 16, no window
    ((400, 90), 4, 2, 128, 1000),            # window beyond every sequence: all zero
])
def test_split_edge_shapes(seqlens, hq, hkv, d, W):
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    q_bits, k_bits = random_qk(int(cu[-1]), hq, hkv, d, seed=int(cu[-1]) + hq)
    scale = 1.0 / math.sqrt(d)
    plain, split = both(q_bits, k_bits, cu, W, scale)
    assert torch.equal(plain, split)
    ref = oracle.future_target(q_bits, k_bits, cu, W, scale)
    got = split.cpu().numpy().astype(np.float64)
    assert float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-3))) <= 2e-3

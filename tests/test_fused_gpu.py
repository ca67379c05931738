"""Single-launch variant (kvpop_future_targets_fused) through the C ABI.

The single launch runs one CTA per work item, the two-launch path CTA pairs
with items twice as tall.  Each row's lse sums the same key tiles in the same
order either way, so lse must be bit-identical to future_targets.  The
transposed pass groups a key's query tiles differently (a pair's second CTA
starts its first query tile 128 rows earlier), so the targets differ only by
fp32 rounding: within 1e-5 relative of the two-launch targets and within the
oracle tolerance; the keep mask must be the oracle's keep mask of the
single launch's own targets.  The small cases are also checked against the
oracle directly.  The flag counters (the workspace before its normaliser
rows) must come back zero-filled after each call so that the workspace can be
reused, and repeated calls must be bit-identical.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import (KvpopError, check_status, fused_workspace, future_targets,
                                           future_targets_fused, target_workspace_bytes)
from future_attention_targets_b200.workloads import make_inputs, random_qk

pytestmark = pytest.mark.gpu
TARGET_TOL = 2e-3


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def rel_err(gpu, ref):
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-3))) if gpu.size else 0.0


def run_both(q_bits, k_bits, cu, W, S, budgets, scale, calls=2):
    q, k = dev(q_bits), dev(k_bits)
    hq, hkv, d = q.shape[1], k.shape[1], q.shape[2]
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = future_targets(q, k, cu, W, S, budgets, scale=scale, status=st2)
    ws = fused_workspace(cu, hq, hkv, d)
    st1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = [future_targets_fused(q, k, cu, W, S, budgets, scale=scale, workspace=ws, status=st1)
            for _ in range(calls)]
    torch.cuda.synchronize()
    check_status(st1)
    check_status(st2)
    counters = ws.numel() - target_workspace_bytes(q.shape[0], hq, hkv, d)
    assert 0 < counters < ws.numel()
    assert int(torch.count_nonzero(ws[:counters])) == 0, "flag counters not cleared by the launch"
    for out in outs:
        for a, b in zip(out, outs[0]):
            assert torch.equal(a, b)
    lse, tgt, keep = outs[-1]
    assert torch.equal(lse, ref[0])
    t, r = tgt.double().cpu().numpy(), ref[1].double().cpu().numpy()
    assert float(np.max(np.abs(t - r) / np.maximum(np.abs(r), 1e-3), initial=0.0)) <= 1e-5
    np.testing.assert_array_equal(keep.cpu().numpy(), oracle.keep_mask(tgt.cpu().numpy(), cu, W, S, budgets))
    return outs[-1]


@pytest.mark.parametrize("name", ["tiny", "qwen3_4b_4k", "varlen_8x"])
def test_fused_matches_two_launch_path(name):
    d = make_inputs(name)
    run_both(d["q_bits"], d["k_bits"], d["cu_seqlens"], d["window"], d["sinks"], d["budgets"], d["scale"])


@pytest.mark.parametrize("seqlens,hq,hkv,d,W", [
    ((300,), 4, 2, 64, 16),                  # head_dim 64
    ((1, 0, 129, 257, 700), 8, 2, 128, 5),   # empty and one-token sequences, ragged tiles
    ((400, 90), 2, 1, 128, 1000),            # window beyond every sequence: targets all zero
    ((2048,), 16, 1, 64, 0),                 # no window, group of 16
])
def test_fused_edge_shapes_against_oracle(seqlens, hq, hkv, d, W):
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T = int(cu[-1])
    q_bits, k_bits = random_qk(T, hq, hkv, d, seed=T + hq)
    scale = 1.0 / math.sqrt(d)
    S = 2
    budgets = [max(S + W, L // 2) for L in seqlens]
    lse, tgt, keep = run_both(q_bits, k_bits, cu, W, S, budgets, scale)
    ref_t = oracle.future_target(q_bits, k_bits, cu, W, scale)
    ref_lse = oracle.row_lse(q_bits, k_bits, cu, scale)
    assert rel_err(tgt.cpu().numpy(), ref_t) <= TARGET_TOL
    assert np.max(np.abs(lse.cpu().numpy() - ref_lse)) <= 2e-4
    assert np.array_equal(keep.cpu().numpy(), oracle.keep_mask(tgt.cpu().numpy(), cu, W, S, budgets))


def test_fused_full_size_16k():
    d = make_inputs("qwen3_8b_16k")
    lse, tgt, keep = run_both(d["q_bits"], d["k_bits"], d["cu_seqlens"], d["window"], d["sinks"], d["budgets"],
                              d["scale"], calls=3)
    assert int(keep.sum()) == 8 * 4032


def test_flag_wait_times_out_and_the_context_survives(monkeypatch):
    """Counters that can never reach their thresholds (a workspace that was not zero-filled, which the
    contract rules out) leave every transposed-pass producer waiting for lse tiles: each wait gives up
    after its limit (50 ms here, through KVPOP_WAIT_NS), the status word reports a timeout, the launch
    ends, and after zero-filling the workspace the same call gives the right results."""
    monkeypatch.setenv("KVPOP_WAIT_NS", "50000000")
    d = make_inputs("tiny")
    q, k = dev(d["q_bits"]), dev(d["k_bits"])
    hq, hkv, hd = q.shape[1], k.shape[1], q.shape[2]
    cu, W, S, budgets, scale = d["cu_seqlens"], d["window"], d["sinks"], d["budgets"], d["scale"]
    ws = fused_workspace(cu, hq, hkv, hd)
    counters = ws.numel() - target_workspace_bytes(q.shape[0], hq, hkv, hd)
    ws[:counters].view(torch.int32).fill_(-(1 << 30))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    future_targets_fused(q, k, cu, W, S, budgets, scale=scale, workspace=ws, status=status)
    with pytest.raises(KvpopError, match="TIMEOUT"):
        check_status(status)
    # A timeout code; the site is the first wait to give up (the flag wait, or a wait downstream of it).
    assert int(status.item()) & 0xff == 4
    ws.zero_()
    status.zero_()
    out = future_targets_fused(q, k, cu, W, S, budgets, scale=scale, workspace=ws, status=status)
    check_status(status)
    ref_t = oracle.future_target(d["q_bits"], d["k_bits"], cu, W, scale)
    assert rel_err(out[1].cpu().numpy(), ref_t) <= TARGET_TOL
    assert torch.equal(out[0], future_targets(q, k, cu, W, S, budgets, scale=scale)[0])

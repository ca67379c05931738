"""The whole path with the most sequences one call accepts (512), ragged.

Per-sequence tables (the level schedule, the single launch's flag-tile bases,
the cache kernels' sequence starts and budgets) all hold 512 entries; every
one is used here, with empty, one-token and window-length sequences among
them.  Targets and lse are compared with the oracle in full, the keep mask,
thresholds and compaction bit for bit, and the single-launch and
host-buffer pipelines must equal the device pipeline.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import (HostPipeline, check_status, compact_kv, future_targets,
                                           future_targets_fused, prefix_topk_thresholds)
from future_attention_targets_b200.workloads import random_qk

pytestmark = pytest.mark.gpu

N_SEQ, HQ, HKV, D, W, S = 512, 4, 2, 64, 16, 2


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def rel_err(gpu, ref):
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-3)))


def test_max_batch_all_entry_points():
    rng = np.random.default_rng(21)
    seqlens = rng.integers(0, 300, N_SEQ)
    seqlens[:6] = [0, 1, W, W + 1, 0, 299]
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T = int(cu[-1])
    budgets = [max(S + W, int(L) // 2) for L in seqlens]
    scale = 1.0 / math.sqrt(D)
    q_bits, k_bits = random_qk(T, HQ, HKV, D, seed=22, gain=2.0)
    q, k = dev(q_bits), dev(k_bits)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    lse, tgt, keep = future_targets(q, k, cu, W, S, budgets, scale=scale, status=status)
    fused = future_targets_fused(q, k, cu, W, S, budgets, scale=scale, status=status)
    check_status(status)
    # The single launch (one CTA per item) sums each row's lse like the two-launch path (CTA pairs) and
    # groups a key's query tiles differently: identical lse, targets equal up to fp32 rounding.
    assert torch.equal(fused[0], lse)
    f_t = fused[1].cpu().numpy()
    assert rel_err(f_t, tgt.cpu().numpy()) <= 1e-5
    np.testing.assert_array_equal(fused[2].cpu().numpy(), oracle.keep_mask(f_t, cu, W, S, budgets))
    tgt_h, keep_h = tgt.cpu().numpy(), keep.cpu().numpy()
    ref_t, ref_l = oracle.future_target(q_bits, k_bits, cu, W, scale, return_lse=True)
    assert rel_err(tgt_h, ref_t) <= 2e-3
    assert float(np.max(np.abs(lse.cpu().numpy() - ref_l))) <= 2e-4
    np.testing.assert_array_equal(keep_h, oracle.keep_mask(tgt_h, cu, W, S, budgets))

    pipe = HostPipeline(cu, HQ, HKV, D, W, S, budgets, scale=scale)
    t_host, k_host = pipe(torch.from_numpy(q_bits.view(np.int16)).view(torch.bfloat16).pin_memory(),
                          torch.from_numpy(k_bits.view(np.int16)).view(torch.bfloat16).pin_memory())
    check_status(pipe.status)
    assert torch.equal(t_host, tgt.cpu()) and torch.equal(k_host, keep.cpu())

    ts, tp = prefix_topk_thresholds(tgt, cu, W, S, budgets)
    rs, rp = oracle.prefix_topk_thresholds(tgt_h, cu, W, S, budgets)
    np.testing.assert_array_equal(tp.cpu().numpy(), rp)
    np.testing.assert_array_equal(ts.cpu().numpy(), rs)

    C = max(budgets)
    v_bits, _ = random_qk(T, HKV, HKV, D, seed=23)
    kc, vc, pos, cnt = compact_kv(k, dev(v_bits), keep, cu, C)
    rk, rv, rpos, rc = oracle.compact_kv(k_bits, v_bits, keep_h, cu, C)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)
    np.testing.assert_array_equal(pos.cpu().numpy(), rpos)
    np.testing.assert_array_equal(kc.cpu().view(torch.int16).numpy().view(np.uint16), rk)
    np.testing.assert_array_equal(vc.cpu().view(torch.int16).numpy().view(np.uint16), rv)

"""The whole path at the longest sequence the library accepts (131,072 tokens).

Small head counts keep it cheap; what is under test is the length: 1024 key
and query tiles per sequence, the deepest level schedule, 128 threshold
blocks per (sequence, KV head), and 1024 compaction slot ranges.
- all-zero keys: A[i, j] = 1/(i+1), so every target and every lse has a
  closed form, checked elementwise over all 131,072 positions;
- random keys with W = 0: each KV head's targets sum to G * L;
- random keys with a window: the targets of the last keys before the window
  and sampled lse rows against the oracle, the keep mask bit for bit, the
  eviction thresholds at sampled steps and the compacted cache bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import (check_status, compact_kv, future_targets, prefix_topk_thresholds)
from future_attention_targets_b200.workloads import random_qk

pytestmark = pytest.mark.gpu

L_MAX = 131072
HQ, HKV, D = 2, 1, 64
TARGET_TOL = 2e-3
LSE_TOL = 2e-4   # the row logsumexp's bound (see test_parity_gpu)


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def rel_err(gpu, ref):
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-3)))


def run(q_bits, k_bits, W, S, budget):
    cu = np.array([0, L_MAX], dtype=np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse, tgt, keep = future_targets(dev(q_bits), dev(k_bits), cu, W, S, [budget], scale=1.0 / math.sqrt(D),
                                    status=status)
    check_status(status)
    return cu, lse, tgt, keep


def test_zero_keys_closed_form_at_max_length():
    W = 1000
    q_bits, k_bits = random_qk(L_MAX, HQ, HKV, D, seed=11, k_zero=True)
    _, lse, tgt, _ = run(q_bits, k_bits, W, 4, 8192)
    inv = 1.0 / np.arange(1, L_MAX + 1, dtype=np.float64)
    tail = np.concatenate([np.cumsum(inv[::-1])[::-1], [0.0]])        # tail[n] = sum_{i >= n} 1/(i+1)
    expect = (HQ // HKV) * tail[np.minimum(np.arange(L_MAX) + W, L_MAX)]
    assert rel_err(tgt.cpu().numpy()[0], expect) <= TARGET_TOL
    assert float(np.max(np.abs(lse.cpu().numpy() - np.log(np.arange(1, L_MAX + 1))[None, :]))) <= LSE_TOL


def test_rows_sum_to_one_at_max_length():
    q_bits, k_bits = random_qk(L_MAX, HQ, HKV, D, seed=12, gain=2.0)
    _, _, tgt, _ = run(q_bits, k_bits, 0, 0, L_MAX)
    np.testing.assert_allclose(tgt.cpu().numpy().astype(np.float64).sum(axis=1), (HQ // HKV) * L_MAX, rtol=1e-4)


def test_random_keys_at_max_length_against_the_oracle():
    W, S, budget = 256, 4, 16384
    scale = 1.0 / math.sqrt(D)
    q_bits, k_bits = random_qk(L_MAX, HQ, HKV, D, seed=13, gain=2.0)
    cu, lse, tgt, keep = run(q_bits, k_bits, W, S, budget)
    tgt_h, keep_h = tgt.cpu().numpy(), keep.cpu().numpy()
    key_lo = L_MAX - W - 384
    ref = oracle.future_target(q_bits, k_bits, cu, W, scale, key_lo=key_lo)
    assert rel_err(tgt_h[0, key_lo:], ref[0, key_lo:]) <= TARGET_TOL
    rows = np.sort(np.random.default_rng(5).choice(L_MAX, size=24, replace=False))
    ref_l = oracle.row_lse(q_bits, k_bits, cu, scale, rows=rows)
    assert float(np.max(np.abs(lse.cpu().numpy()[:, rows] - ref_l[:, rows]))) <= LSE_TOL
    np.testing.assert_array_equal(keep_h, oracle.keep_mask(tgt_h, cu, W, S, [budget]))
    assert int(keep_h.sum()) == budget

    steps = np.concatenate([np.arange(0, 4), [budget - 2, budget - 1, budget, budget + 1],
                            np.random.default_rng(6).choice(L_MAX, size=60, replace=False), [L_MAX - 1]])
    ts, tp = prefix_topk_thresholds(tgt, cu, W, S, [budget])
    rs, rp = oracle.prefix_topk_thresholds(tgt_h, cu, W, S, [budget], steps=steps)
    ts_h, tp_h = ts.cpu().numpy(), tp.cpu().numpy()
    for t in steps:
        assert tp_h[0, t] == rp[0, t], t
        assert (ts_h[0, t] == rs[0, t]) or (np.isnan(ts_h[0, t]) and np.isnan(rs[0, t])), t

    v_bits, _ = random_qk(L_MAX, HKV, HKV, D, seed=14)
    kc, vc, pos, cnt = compact_kv(dev(k_bits), dev(v_bits), keep, cu, budget)
    rk, rv, rp2, rc = oracle.compact_kv(k_bits, v_bits, keep_h, cu, budget)
    np.testing.assert_array_equal(kc.cpu().view(torch.int16).numpy().view(np.uint16), rk)
    np.testing.assert_array_equal(vc.cpu().view(torch.int16).numpy().view(np.uint16), rv)
    np.testing.assert_array_equal(pos.cpu().numpy(), rp2)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)

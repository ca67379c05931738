"""Seeded random problems through the whole hot path and its downstream rows, against the oracle.

Each case draws (from a fixed seed) a batch of ragged sequences, a GQA shape, a head dimension, a
window, sinks, budgets and an input gain (gains up to 6 send many of pass 1's tiles down its exact
path); a few long cases (1-2 sequences of 2,000-6,000 tokens, gains 4 and 6) give rows many key tiles
whose scores can jump far above the running offset.  Each case checks:
- lse within 2e-4 and every target within 2e-3 (floor 1e-3) of the fp64 oracle;
- the keep mask bit-exact against the oracle's mask from the same fp32 targets;
- the prefix top-k thresholds bit-exact;
- the compacted cache bit-exact and one decode step within 2e-3 (global reading) of the oracle;
- the same results from the separate calls (row_lse, future_target, keep_mask) as from the pipeline,
  and from the single launch the same lse bits, its targets against the oracle and its keep mask exact.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import _binding as B
from future_attention_targets_b200.workloads import random_qk

pytestmark = pytest.mark.gpu

TARGET_TOL, LSE_TOL = 2e-3, 2e-4
N_CASES = 40


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


N_LONG = 4   # cases with fewer, longer sequences (many key tiles per row), large gains among them


def draw(seed):
    rng = np.random.default_rng(1000 + seed)
    long_case = seed >= N_CASES
    nb = int(rng.integers(1, 3 if long_case else 6))
    seqlens = [int(x) for x in rng.integers(2000 if long_case else 0, 6000 if long_case else 1300, nb)]
    if sum(seqlens) == 0:
        seqlens[0] = 1
    hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4, 8]))
    d = int(rng.choice([64, 128]))
    W = int(rng.choice([0, 1, 16, 100, 256, 700]))
    S = int(rng.integers(0, 5))
    budgets = [W + S + int(rng.integers(0, 400)) for _ in seqlens]
    gain = float(rng.choice([4.0, 6.0] if long_case else [0.5, 1.0, 2.0, 4.0, 6.0]))
    if long_case:
        hkv, G = 1, int(rng.choice([1, 2, 4]))
    return seqlens, hkv * G, hkv, d, W, S, budgets, gain


@pytest.mark.parametrize("seed", range(N_CASES + N_LONG))
def test_random_problem(seed):
    seqlens, hq, hkv, d, W, S, budgets, gain = draw(seed)
    T = sum(seqlens)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    scale = 1.0 / math.sqrt(d)
    q_bits, k_bits = random_qk(T, hq, hkv, d, seed=seed, gain=gain)
    q, k = dev(q_bits), dev(k_bits)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    lse, tgt, keep = B.future_targets(q, k, cu, W, S, budgets, scale=scale, status=st)
    B.check_status(st)
    ref_t, ref_l = oracle.future_target(q_bits, k_bits, cu, W, scale, return_lse=True)
    lse_h, tgt_h, keep_h = lse.cpu().numpy(), tgt.cpu().numpy(), keep.cpu().numpy()
    assert float(np.max(np.abs(lse_h.astype(np.float64) - ref_l), initial=0.0)) <= LSE_TOL
    err = np.abs(tgt_h.astype(np.float64) - ref_t) / np.maximum(np.abs(ref_t), 1e-3)
    assert float(np.max(err, initial=0.0)) <= TARGET_TOL
    np.testing.assert_array_equal(keep_h, oracle.keep_mask(tgt_h, cu, W, S, budgets))

    # The single launch (one CTA per SM, both passes): the same lse bits; its targets against the oracle
    # like the pipeline's (its 128-key blocks align query tiles differently, so an element may take the
    # polynomial in one path and MUFU in the other: they differ by up to the polynomial's 8.6e-5), and
    # its own keep mask exact.
    lf, tf, kf = B.future_targets_fused(q, k, cu, W, S, budgets, scale=scale, status=st)
    B.check_status(st)
    assert torch.equal(lf, lse)
    tf_h = tf.cpu().numpy()
    errf = np.abs(tf_h.astype(np.float64) - ref_t) / np.maximum(np.abs(ref_t), 1e-3)
    assert float(np.max(errf, initial=0.0)) <= TARGET_TOL
    np.testing.assert_array_equal(kf.cpu().numpy(), oracle.keep_mask(tf_h, cu, W, S, budgets))

    # The separate calls give the same bits as the pipeline.
    l2 = B.row_lse(q, k, cu, scale, status=st)
    t2 = B.future_target(q, k, cu, W, l2, scale, status=st)
    k2 = B.keep_mask(t2, cu, W, S, budgets)
    B.check_status(st)
    assert torch.equal(l2, lse) and torch.equal(t2, tgt) and torch.equal(k2, keep)

    ts, tp = B.prefix_topk_thresholds(tgt, cu, W, S, budgets)
    rs, rp = oracle.prefix_topk_thresholds(tgt_h, cu, W, S, budgets)
    np.testing.assert_array_equal(tp.cpu().numpy(), rp)
    np.testing.assert_array_equal(ts.cpu().numpy(), rs)

    C = max(max(budgets), 1)
    v_bits, _ = random_qk(T, hkv, hkv, d, seed=seed + 77)
    kc, vc, pos, cnt = B.compact_kv(k, dev(v_bits), keep, cu, C)
    rk, rv, rpos, rc = oracle.compact_kv(k_bits, v_bits, keep_h, cu, C)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)
    np.testing.assert_array_equal(pos.cpu().numpy(), rpos)
    np.testing.assert_array_equal(kc.cpu().view(torch.int16).numpy(), rk.view(np.int16))
    np.testing.assert_array_equal(vc.cpu().view(torch.int16).numpy(), rv.view(np.int16))
    if G_ok(hq // hkv):
        nb = len(seqlens)
        qd_bits, _ = random_qk(nb, hq, hkv, d, seed=seed + 78)
        out, _ = B.decode_attention(dev(qd_bits.reshape(nb, hq, d)), kc, vc, cnt, scale)
        ro, _ = oracle.decode_attention(qd_bits.reshape(nb, hq, d), rk, rv, rc, scale)
        o = out.cpu().numpy().astype(np.float64)
        assert float(np.max(np.abs(o - ro), initial=0.0)) <= TARGET_TOL * max(float(np.max(np.abs(ro), initial=0.0)),
                                                                              1e-3)


def G_ok(G):
    return G <= 16 and G & (G - 1) == 0

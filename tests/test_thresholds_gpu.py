"""Prefix top-k eviction thresholds: the CUDA kernel (through the C ABI)
against the CPU oracle.  Positions must match exactly and scores bit for bit
(both sides only select among the input values)."""
import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import keep_mask, prefix_topk_thresholds

pytestmark = pytest.mark.gpu


def run(score, cu, W, S, budgets):
    ts, tp = prefix_topk_thresholds(torch.from_numpy(np.ascontiguousarray(score)).cuda(), cu, W, S, budgets)
    return ts.cpu().numpy(), tp.cpu().numpy()


def assert_same(got, ref):
    np.testing.assert_array_equal(got[1], ref[1])
    np.testing.assert_array_equal(got[0], ref[0])


CASES = [
    # seqlens, H_kv, W, S, scored slots per sequence, score kind
    ((200,), 2, 16, 4, [40], "uniform"),
    ((12, 400, 37, 250), 3, 16, 4, [10, 100, 60, 0], "ties"),
    ((3000,), 1, 32, 4, [700], "uniform"),        # several 1024-step blocks
    ((2500,), 2, 8, 2, [2000], "ties"),           # k larger than a block
    ((9000,), 1, 4, 4, [8192], "uniform"),        # the largest k
    ((1500, 1, 2100), 2, 64, 0, [300, 5, 1], "special"),
    ((20000,), 1, 16, 4, [10000], "uniform"),     # k beyond 8192: the band is taken from a large K
    ((6000, 3000), 2, 8, 4, [1500, 2900], "coarse"),   # four distinct scores: ties across the band edges
    ((5000,), 1, 8, 4, [1024], "coarse"),         # band of exactly kBlock + 1 with k near a block
]


def make_scores(kind, H, T, seed):
    rng = np.random.default_rng(seed)
    s = rng.random((H, T)).astype(np.float32)
    if kind == "ties":
        s = np.round(s * 16) / 16
    if kind == "coarse":
        s = np.floor(s * 4) / 4
    if kind == "special":
        s[:, ::11] = 0.5
        s[0, 5::97] = np.nan
        s[0, 7::89] = -0.0
        s[0, 9::83] = 0.0
        s[-1, 3::71] = np.inf
        s[-1, 4::73] = -np.inf
    return s.astype(np.float32)


@pytest.mark.parametrize("case", CASES, ids=[f"L{c[0]}-k{c[4]}-{c[5]}" for c in CASES])
def test_thresholds_match_oracle(case):
    seqlens, H, W, S, slots, kind = case
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    budgets = [S + W + k for k in slots]
    score = make_scores(kind, H, int(cu[-1]), seed=sum(seqlens))
    assert_same(run(score, cu, W, S, budgets), oracle.prefix_topk_thresholds(score, cu, W, S, budgets))


def test_thresholds_16k_sampled_and_consistent():
    """At the 16k size: sampled steps against the oracle, monotone thresholds,
    and the last step keeps exactly the keep mask's scored tokens."""
    L, H, W, S, budget = 16384, 8, 256, 4, 4032
    rng = np.random.default_rng(3)
    score = (rng.random((H, L)) ** 3).astype(np.float32)
    cu = np.array([0, L], dtype=np.int32)
    ts, tp = run(score, cu, W, S, [budget])
    steps = list(range(0, L, 997)) + list(range(L - 40, L)) + [S + W + budget - S - W - 1 + d for d in range(-2, 3)]
    rs, rp = oracle.prefix_topk_thresholds(score[:2], cu, W, S, [budget], steps=steps)
    sel = np.array(sorted(set(s for s in steps if 0 <= s < L)))
    np.testing.assert_array_equal(tp[:2, sel], rp[:, sel])
    np.testing.assert_array_equal(ts[:2, sel], rs[:, sel])
    keep = keep_mask(torch.from_numpy(score).cuda(), cu, W, S, [budget]).cpu().numpy()
    for h in range(H):
        defined = tp[h] >= 0
        key = np.where(defined, ts[h].astype(np.float64), -np.inf)
        # monotone in the keep order: score never decreases; on equal score the position never increases
        d_s = np.diff(key[defined])
        d_p = np.diff(tp[h][defined])
        assert np.all((d_s > 0) | ((d_s == 0) & (d_p <= 0)))
        t_last, p_thr, s_thr = L - 1, tp[h, L - 1], ts[h, L - 1]
        mid = np.arange(S, L - W)
        kept = (score[h, mid] > s_thr) | ((score[h, mid] == s_thr) & (mid <= p_thr))
        np.testing.assert_array_equal(kept.astype(np.uint8), keep[h, S:L - W])

"""Pins for the CPU oracle: checks against facts other than the oracle itself.

Each ``pin_*`` function takes an oracle module (the real one, or a copy with
a planted mistake) and raises AssertionError when the oracle disagrees with
what the definition, the mathematics or the pages fix.  ``test_oracle_pins``
runs them on the real oracle; ``test_oracle_mutants`` checks that every
planted mistake is caught by at least one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from future_attention_targets_b200.workloads import bf16_bits_to_f32, random_qk

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ------------------------------------------------------------ brute force

def brute_force(q, k, cu, W, scale):
    """Scalar triple loop with math.exp / math.fsum: lse [Hq,T], target [Hkv,T], far [Hq,T]."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    lse = [[0.0] * T for _ in range(Hq)]
    far = [[0.0] * T for _ in range(Hq)]
    terms = [[[] for _ in range(T)] for _ in range(Hkv)]
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        for g in range(Hq):
            h = g // G
            for i in range(s, e):
                logits = []
                for j in range(s, i + 1):
                    logits.append(scale * math.fsum(float(q[i, g, t]) * float(k[j, h, t]) for t in range(d)))
                m = max(logits)
                Z = math.fsum(math.exp(x - m) for x in logits)
                lse[g][i] = m + math.log(Z)
                far_terms = []
                for jj, x in enumerate(logits):
                    j = s + jj
                    if i - j >= W:
                        a = math.exp(x - m) / Z
                        terms[h][j].append(a)
                        far_terms.append(a)
                far[g][i] = math.fsum(far_terms)
    target = np.array([[math.fsum(terms[h][j]) for j in range(T)] for h in range(Hkv)])
    return np.array(lse), target, np.array(far)


def _tiny_case(seed, seqlens=(7, 13), Hkv=2, G=2, d=6):
    q_bits, k_bits = random_qk(sum(seqlens), Hkv * G, Hkv, d, seed, gain=2.0)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    return q_bits, k_bits, cu


def pin_brute_force(orc):
    for seed, W in [(1, 0), (2, 1), (3, 5), (4, 12), (5, 13), (6, 40)]:
        q_bits, k_bits, cu = _tiny_case(seed)
        q = bf16_bits_to_f32(q_bits).astype(np.float64)
        k = bf16_bits_to_f32(k_bits).astype(np.float64)
        scale = 1.0 / math.sqrt(q.shape[2])
        lse_b, tgt_b, far_b = brute_force(q, k, cu, W, scale)
        tgt, lse, far = orc.future_target(q_bits, k_bits, cu, W, scale, return_lse=True, return_far=True)
        np.testing.assert_allclose(tgt, tgt_b, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse, lse_b, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(far, far_b, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(orc.row_lse(q_bits, k_bits, cu, scale), lse_b, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------ closed forms

def harmonic_target(L, W, G):
    """All logits equal => A[i, j] = 1/(i+1); target_j = G * sum_{i=j+W}^{L-1} 1/(i+1)."""
    inv = 1.0 / np.arange(1, L + 1, dtype=np.float64)
    tail = np.concatenate([np.cumsum(inv[::-1])[::-1], [0.0]])     # tail[m] = sum_{i>=m} 1/(i+1)
    return G * np.array([tail[min(j + W, L)] for j in range(L)])


def pin_closed_form_zero_keys(orc):
    seqlens = (300, 517)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    for W, which in [(0, "k"), (64, "k"), (5, "q"), (299, "k")]:
        q_bits, k_bits = random_qk(sum(seqlens), 4, 2, 16, seed=7,
                                   q_zero=(which == "q"), k_zero=(which == "k"))
        tgt, lse = orc.future_target(q_bits, k_bits, cu, W, 0.25, return_lse=True)
        for b, L in enumerate(seqlens):
            s = int(cu[b])
            for h in range(2):
                np.testing.assert_allclose(tgt[h, s:s + L], harmonic_target(L, W, 2), rtol=1e-12, atol=1e-15)
            np.testing.assert_allclose(lse[:, s:s + L], np.log(np.arange(1, L + 1))[None, :].repeat(4, 0),
                                       rtol=1e-13, atol=1e-13)


def pin_gqa_grouping(orc):
    """Query heads g // G map to KV head h: zero queries in group 1 force its closed form."""
    T, Hkv, G, d, W = 200, 2, 2, 8, 10
    q_bits, k_bits = random_qk(T, Hkv * G, Hkv, d, seed=11, gain=3.0)
    q_bits = q_bits.copy()
    q_bits[:, 2:4, :] = 0                                  # heads 2, 3 = group of KV head 1
    cu = np.array([0, T], dtype=np.int32)
    tgt = orc.future_target(q_bits, k_bits, cu, W, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(tgt[1], harmonic_target(T, W, G), rtol=1e-12, atol=1e-15)
    assert not np.allclose(tgt[0], harmonic_target(T, W, G), rtol=1e-3)


def pin_row_stochastic(orc):
    """W = 0: every query row sums to 1, so the targets of a KV head sum to G * L."""
    seqlens = (33, 90)
    q_bits, k_bits = random_qk(sum(seqlens), 6, 3, 16, seed=5, gain=4.0)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    tgt = orc.future_target(q_bits, k_bits, cu, 0, 0.25)
    for b, L in enumerate(seqlens):
        s = int(cu[b])
        np.testing.assert_allclose(tgt[:, s:s + L].sum(axis=1), 2 * L, rtol=1e-12)
    # W >= L: nothing has left the window.
    tgt = orc.future_target(q_bits, k_bits, cu, 90, 0.25)
    assert np.all(tgt[:, cu[1]:] == 0) and np.all(tgt[:, :cu[1]] == 0)


def pin_mass_conservation(orc):
    """sum_j target[h, j] = sum_{g in group(h)} sum_i far[g, i], and target = 0 for j >= L - W."""
    seqlens = (150, 61)
    q_bits, k_bits = random_qk(sum(seqlens), 8, 2, 16, seed=9, gain=3.0)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    W = 20
    tgt, far = orc.future_target(q_bits, k_bits, cu, W, 0.3, return_far=True)
    for b, L in enumerate(seqlens):
        s = int(cu[b])
        for h in range(2):
            np.testing.assert_allclose(tgt[h, s:s + L].sum(), far[4 * h:4 * h + 4, s:s + L].sum(), rtol=1e-12)
            assert np.all(tgt[h, s + L - W:s + L] == 0)
            assert np.all(tgt[h, s:s + L - W] > 0)


def pin_single_token(orc):
    """L = 1: the row holds one term, lse = s q.k exactly."""
    q_bits, k_bits = random_qk(1, 2, 1, 8, seed=3, gain=2.0)
    cu = np.array([0, 1], dtype=np.int32)
    q = bf16_bits_to_f32(q_bits).astype(np.float64)
    k = bf16_bits_to_f32(k_bits).astype(np.float64)
    lse = orc.row_lse(q_bits, k_bits, cu, 0.7)
    for g in range(2):
        assert abs(lse[g, 0] - 0.7 * float(q[0, g] @ k[0, 0])) < 1e-14
    tgt = orc.future_target(q_bits, k_bits, cu, 0, 0.7)
    assert abs(tgt[0, 0] - 2.0) < 1e-14                   # each head's row is that one key


def pin_dominant_key(orc):
    """A key with a huge logit for every later query takes ~all of their mass."""
    T, d, W, jstar = 120, 16, 7, 30
    rng = np.random.default_rng(4)
    v = np.ones(d)
    q = np.tile(v, (T, 2, 1)) + 0.01 * rng.standard_normal((T, 2, d))
    k = 0.01 * rng.standard_normal((T, 1, d))
    k[jstar, 0] = 8.0 * v
    cu = np.array([0, T], dtype=np.int32)
    tgt = orc.future_target(q, k, cu, W, 1.0)
    expect = 2.0 * (T - jstar - W)
    assert abs(tgt[0, jstar] - expect) < 1e-6 * expect
    # Queries at or after j* give (almost) nothing to earlier keys: their targets
    # equal those of the sequence cut just before j*.
    cut = orc.future_target(q[:jstar], k[:jstar], np.array([0, jstar], dtype=np.int32), W, 1.0)
    np.testing.assert_allclose(tgt[0, :jstar], cut[0], rtol=0, atol=1e-6)


# ------------------------------------------------------------ keep mask

def keep_mask_by_sorting(score, cu, W, S, budgets):
    """Independent ranking: Python's sorted() on (nan-flag, -score, position)."""
    Hkv, T = score.shape
    keep = np.zeros((Hkv, T), dtype=np.uint8)
    for b in range(len(cu) - 1):
        s, L = int(cu[b]), int(cu[b + 1] - cu[b])
        B = int(budgets[b])
        for h in range(Hkv):
            if L <= B:
                keep[h, s:s + L] = 1
                continue
            cand = []
            for p in range(S, L - W):
                x = float(score[h, s + p])
                cand.append((1 if math.isnan(x) else 0, 0.0 if math.isnan(x) else -x, p))
            for _, _, p in sorted(cand)[:B - S - W]:
                keep[h, s + p] = 1
            keep[h, s:s + S] = 1
            keep[h, s + L - W:s + L] = 1
    return keep


def pin_keep_mask(orc):
    rng = np.random.default_rng(21)
    seqlens = (12, 400, 37, 250, 300)                    # the first is shorter than sinks + window
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T = int(cu[-1])
    W, S = 16, 4
    budgets = np.array([30, 100, 60, 250, 20], dtype=np.int32)
    score = rng.random((3, T)).astype(np.float32)
    score[0, ::7] = 0.5                                   # many exact ties
    score[1, 62:162] = 2.0                                # 100 tied top scores, k = 80: the tie rule decides
    score[2, 22] = np.nan
    score[2, 23] = -0.0
    score[2, 24] = 0.0
    score[2, 25] = np.inf
    got = orc.keep_mask(score, cu, W, S, budgets)
    ref = keep_mask_by_sorting(score, cu, W, S, budgets)
    np.testing.assert_array_equal(got, ref)
    for b, L in enumerate(seqlens):
        s = int(cu[b])
        assert np.all(got[:, s:s + L].sum(axis=1) == min(int(budgets[b]), L))
        if L > budgets[b]:
            mid = slice(s + S, s + L - W)
            for h in range(3):
                kept = score[h, mid][got[h, mid] == 1]
                drop = score[h, mid][got[h, mid] == 0]
                kept, drop = kept[~np.isnan(kept)], drop[~np.isnan(drop)]
                if len(kept) and len(drop):
                    assert kept.min() >= drop.max()


def pin_budget_from_pages(orc):
    """The model card's 16k budget: 4 + 3,772 + 256 = 4,032 kept per head."""
    with open(os.path.join(GOLDEN, "kvpop_budget_16k.json")) as f:
        g = json.load(f)
    assert g["sinks"] + g["scored_top_k"] + g["recent_window"] == g["entries_per_head"]
    assert g["context"] // 4 == g["quarter_of_context"] == g["entries_per_head"] + g["reserved_for_scorer_memory"]
    L = g["context"]
    rng = np.random.default_rng(0)
    score = rng.random((2, L))
    cu = np.array([0, L], dtype=np.int32)
    keep = orc.keep_mask(score, cu, g["recent_window"], g["sinks"], [g["entries_per_head"]])
    assert np.all(keep.sum(axis=1) == g["entries_per_head"])
    assert np.all(keep[:, :g["sinks"]] == 1) and np.all(keep[:, L - g["recent_window"]:] == 1)
    mid = keep[:, g["sinks"]:L - g["recent_window"]]
    assert np.all(mid.sum(axis=1) == g["scored_top_k"])


def pin_keep_protected_positions(orc):
    """The scored top-k is drawn only from [S, L - W): sinks and recent-window
    tokens are kept by position, so giving them the highest scores must not
    let them take a scored slot (model card introduction: sinks, scored older
    tokens and recent tokens each have their own share of the budget)."""
    W, S = 5, 3
    seqlens = (40, 25, 21)                        # L = budget + 1 in the last: exactly one token evicted
    budgets = [20, 14, 20]
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    rng = np.random.default_rng(5)
    score = rng.random((2, int(cu[-1]))).astype(np.float32)
    for b, L in enumerate(seqlens):
        s = int(cu[b])
        score[:, s:s + S] = np.inf                 # sinks score highest
        score[0, s + L - W:s + L] = 1e30           # so does the whole recent window
        score[1, s + L - W] = 1e30                 # only its first position (the candidate range's edge)
    got = orc.keep_mask(score, cu, W, S, budgets)
    np.testing.assert_array_equal(got, keep_mask_by_sorting(score, cu, W, S, budgets))
    for b, L in enumerate(seqlens):
        s = int(cu[b])
        assert np.all(got[:, s:s + L].sum(axis=1) == budgets[b])
        assert np.all(got[:, s + S:s + L - W].sum(axis=1) == budgets[b] - S - W)


# ------------------------------------------------------------ restrictions

def pin_restrictions(orc):
    """key_lo / rows restrictions agree with the full computation where defined."""
    seqlens = (140, 333)
    q_bits, k_bits = random_qk(sum(seqlens), 4, 2, 16, seed=13, gain=2.0)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    W = 9
    full, lse = orc.future_target(q_bits, k_bits, cu, W, 0.3, return_lse=True)
    part = orc.future_target(q_bits, k_bits, cu, W, 0.3, key_lo=100)
    for b, L in enumerate(seqlens):
        s = int(cu[b])
        assert np.all(np.isnan(part[:, s:s + 100]))
        np.testing.assert_allclose(part[:, s + 100:s + L], full[:, s + 100:s + L], rtol=1e-13, atol=1e-16)
    rows = np.array([0, 5, 139, 140, 141, 300, 472])
    lr = orc.row_lse(q_bits, k_bits, cu, 0.3, rows=rows)
    np.testing.assert_allclose(lr[:, rows], lse[:, rows], rtol=1e-13)


ALL_PINS = [
    pin_brute_force,
    pin_closed_form_zero_keys,
    pin_gqa_grouping,
    pin_row_stochastic,
    pin_mass_conservation,
    pin_single_token,
    pin_dominant_key,
    pin_keep_mask,
    pin_budget_from_pages,
    pin_keep_protected_positions,
    pin_restrictions,
]


# ------------------------------------------------------------ prefix top-k thresholds

def online_eviction(score_row, L, W, S, k_top):
    """Token-by-token online eviction with a heap (independent of the oracle):
    the scored slots hold at most k_top of the tokens that have left the
    window; when they overflow, the worst (lowest score, then larger position,
    NaN lowest) is evicted.  Returns the kept set after each step."""
    import heapq
    heap, kept, evicted, out = [], set(), set(), []
    for t in range(L):
        p = t - W
        if p >= S:
            x = float(score_row[p])
            # heap entry orders "worse" first: (nan flag inverted, score, -position)
            key = (0 if math.isnan(x) else 1, 0.0 if math.isnan(x) else x, -p)
            heapq.heappush(heap, (key, p))
            kept.add(p)
            while len(kept) > k_top:
                _, q = heapq.heappop(heap)
                kept.discard(q)
                evicted.add(q)
        out.append(set(kept))
    return out


def _rank_at_or_above(x, p, ts, tp):
    """(x, p) ranks at or above the threshold (ts, tp) in the keep-set order."""
    xn, tn = math.isnan(x), math.isnan(ts)
    if tn and xn:
        return p <= tp
    if tn:
        return True
    if xn:
        return False
    return x > ts or (x == ts and p <= tp)


def pin_prefix_thresholds(orc):
    rng = np.random.default_rng(31)
    seqlens = (70, 9, 130, 45)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T = int(cu[-1])
    W, S = 6, 3
    budgets = [W + S + 10, W + S + 3, W + S + 25, W + S]          # last: k = 0
    score = rng.random((2, T)).astype(np.float32)
    score[0, ::5] = 0.25                                          # ties
    score[1, 20:40] = 0.75
    score[1, 50] = np.nan
    thr_s, thr_p = orc.prefix_topk_thresholds(score, cu, W, S, budgets)
    keep_final = orc.keep_mask(score, cu, W, S, budgets)
    for b, L in enumerate(seqlens):
        s0 = int(cu[b])
        k_top = budgets[b] - S - W
        for h in range(2):
            sets = online_eviction(score[h, s0:s0 + L], L, W, S, k_top)
            for t in range(L):
                ts, tp = float(thr_s[h, s0 + t]), int(thr_p[h, s0 + t])
                cand = range(S, t - W + 1) if t - W >= S else range(0)
                if tp == -1 and ts == -np.inf:
                    assert sets[t] == set(cand)                  # nothing evicted yet
                    continue
                kept = {p for p in cand if _rank_at_or_above(float(score[h, s0 + p]), p, ts, tp)}
                assert kept == sets[t], (b, h, t)
                if k_top > 0:
                    assert len(kept) == k_top and tp in kept
            # monotone: once defined, the threshold never gets worse
            prev = None
            for t in range(L):
                ts, tp = float(thr_s[h, s0 + t]), int(thr_p[h, s0 + t])
                if tp < 0:
                    continue
                if prev is not None:
                    assert _rank_at_or_above(ts, tp, *prev)
                prev = (ts, tp)
            # the last step agrees with the keep mask's scored slots
            if L > budgets[b] and L - 1 - W >= S:
                ts, tp = float(thr_s[h, s0 + L - 1]), int(thr_p[h, s0 + L - 1])
                mid = [p for p in range(S, L - W) if keep_final[h, s0 + p]]
                assert set(mid) == sets[L - 1]


ALL_PINS.append(pin_prefix_thresholds)


def pin_threshold_steps(orc):
    """The steps= restriction agrees with the full computation."""
    rng = np.random.default_rng(8)
    cu = np.array([0, 60, 200], dtype=np.int32)
    score = rng.random((2, 200)).astype(np.float32)
    full_s, full_p = orc.prefix_topk_thresholds(score, cu, 5, 2, [17, 40])
    steps = [0, 6, 7, 30, 59, 100, 139]
    part_s, part_p = orc.prefix_topk_thresholds(score, cu, 5, 2, [17, 40], steps=steps)
    for b in range(2):
        s0, L = int(cu[b]), int(cu[b + 1] - cu[b])
        for t in range(L):
            if t in steps:
                assert part_p[0, s0 + t] == full_p[0, s0 + t] and part_p[1, s0 + t] == full_p[1, s0 + t]
                np.testing.assert_array_equal(part_s[:, s0 + t], full_s[:, s0 + t])
            else:
                assert np.all(part_p[:, s0 + t] == -2)


ALL_PINS.append(pin_threshold_steps)



def pin_threshold_onset(orc):
    """The steps where the threshold starts to exist.  With k = budget - S - W
    scored slots, step t has t - W - S + 1 candidates.  While fewer than k
    compete nothing is evicted: (-inf, -1).  At the step where exactly k
    compete the threshold is the k-th best of them, i.e. the worst one in the
    keep order (computed here with sorted()).  With k = 0 the first candidate
    already makes it (+inf, -1): nothing is kept."""
    W, S = 4, 2
    budgets = [W + S + 6, W + S, W + S + 1]
    seqlens = (30, 12, 20)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    rng = np.random.default_rng(17)
    score = rng.random((2, int(cu[-1]))).astype(np.float32)
    score[1, :] = 0.5                                  # all tied: position order decides
    thr_s, thr_p = orc.prefix_topk_thresholds(score, cu, W, S, budgets)
    for b, L in enumerate(seqlens):
        s0, k_top = int(cu[b]), budgets[b] - S - W
        onset = S + W + max(k_top, 1) - 1              # first step with max(k, 1) candidates
        for h in range(2):
            for t in range(onset):
                assert thr_s[h, s0 + t] == -np.inf and thr_p[h, s0 + t] == -1, (b, h, t)
            if k_top == 0:
                assert thr_s[h, s0 + onset] == np.inf and thr_p[h, s0 + onset] == -1
                continue
            cand = sorted((-float(score[h, s0 + p]), p) for p in range(S, onset - W + 1))
            assert len(cand) == k_top
            worst = cand[-1]
            assert thr_p[h, s0 + onset] == worst[1] and thr_s[h, s0 + onset] == -worst[0], (b, h)


def pin_budget_below_protected(orc):
    """A budget smaller than sinks + window leaves no room for the protected
    tokens; both the keep mask and the thresholds reject it."""
    cu = np.array([0, 50], dtype=np.int32)
    score = np.zeros((1, 50), dtype=np.float32)
    for fn in (orc.keep_mask, orc.prefix_topk_thresholds):
        try:
            fn(score, cu, 8, 4, [11])
        except ValueError:
            pass
        else:
            raise AssertionError(f"{fn.__name__} accepted a budget below sinks + window")
        fn(score, cu, 8, 4, [12])                      # exactly sinks + window is allowed


ALL_PINS.extend([pin_threshold_onset, pin_budget_below_protected])


# ------------------------------------------------------------ static cache: compaction + decode attention

def pin_compact_kv(orc):
    rng = np.random.default_rng(12)
    seqlens = (30, 0, 45)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T, Hkv, d = int(cu[-1]), 2, 4
    k = rng.integers(0, 2**16, size=(T, Hkv, d)).astype(np.uint16)
    v = rng.integers(0, 2**16, size=(T, Hkv, d)).astype(np.uint16)
    keep = (rng.random((Hkv, T)) < 0.4).astype(np.uint8)
    kc, vc, pos, cnt = orc.compact_kv(k, v, keep, cu, capacity=15)
    for b, L in enumerate(seqlens):
        s0 = int(cu[b])
        for h in range(Hkv):
            kept = [p for p in range(L) if keep[h, s0 + p]]          # scalar walk, position order
            assert cnt[b, h] == len(kept)
            for slot in range(15):
                if slot < len(kept):
                    p = kept[slot]
                    assert pos[b, h, slot] == p
                    assert list(kc[b, h, slot]) == list(k[s0 + p, h]) and list(vc[b, h, slot]) == list(v[s0 + p, h])
                else:
                    assert pos[b, h, slot] == -1 and not kc[b, h, slot].any() and not vc[b, h, slot].any()


def pin_decode_attention(orc):
    rng = np.random.default_rng(13)
    B, Hq, Hkv, C, d = 2, 4, 2, 9, 5
    q = rng.standard_normal((B, Hq, d))
    kc = rng.standard_normal((B, Hkv, C, d))
    vc = rng.standard_normal((B, Hkv, C, d))
    cnt = np.array([[9, 4], [1, 0]], dtype=np.int32)
    out, lse = orc.decode_attention(q, kc, vc, cnt, 0.6)
    for b in range(B):
        for g in range(Hq):
            h, n = g // 2, int(cnt[b, g // 2])
            if n == 0:
                assert np.all(out[b, g] == 0) and lse[b, g] == -np.inf
                continue
            logits = [0.6 * math.fsum(q[b, g, t] * kc[b, h, s, t] for t in range(d)) for s in range(n)]
            m = max(logits)
            Z = math.fsum(math.exp(x - m) for x in logits)
            for t in range(d):
                ref = math.fsum(math.exp(logits[s] - m) / Z * vc[b, h, s, t] for s in range(n))
                assert abs(out[b, g, t] - ref) < 1e-12
            assert abs(lse[b, g] - (m + math.log(Z))) < 1e-12
    # zero keys: uniform weights, the output is the mean of the filled value rows
    out0, _ = orc.decode_attention(q, np.zeros_like(kc), vc, cnt, 0.6)
    np.testing.assert_allclose(out0[0, 0], vc[0, 0, :9].mean(axis=0), rtol=1e-13)
    np.testing.assert_allclose(out0[0, 2], vc[0, 1, :4].mean(axis=0), rtol=1e-13)
    # one filled slot: the output is that value row
    np.testing.assert_allclose(out[1, 0], vc[1, 0, 0], rtol=1e-13)


ALL_PINS.extend([pin_compact_kv, pin_decode_attention])

"""CPU oracle for KVpop future-attention targets.  TEST INFRASTRUCTURE ONLY.

Only the tests, the package's ``smoke()`` check and ``bench.py``'s CPU
baseline may import this module.  The CUDA library never calls it, and it
shares no code, constants or helpers with the CUDA path.

It is the plain definition written out in float64, with an explicitly
materialised causal softmax (one block of query rows at a time):

* Row logsumexp.  For query head g and query position i of a sequence,
  ``lse[g, i] = log sum_{j <= i} exp(s * q_{g,i} . k_{h(g),j})`` with the
  causal mask (attention from a query only to itself and earlier keys) and
  the GQA mapping ``h(g) = g // G``, ``G = H_q / H_kv``.
* Future-attention target (KVpop paper summary; the aiweekly article
  "KVpop shrinks Qwen3 KV cache 88%", second paragraph; its French
  edition, second paragraph).  Key j is labelled with the softmax
  probability that queries give it once it is outside the window of the W
  most recent positions.  At query i the window holds positions
  i-W+1 .. i, so key j has left it exactly when i >= j + W.  The mass is
  the softmax probability ``A[i, j] = exp(S[i, j] - lse[i])`` and the
  target of a KV head is summed over the G query heads that share it:
  ``target[h, j] = sum_{g in group(h)} sum_{i = j+W}^{L-1} A_g[i, j]``.
* Keep mask (KVpop model card, introduction: the cache is bounded and made
  of initial sink tokens, scored older tokens and recent tokens, with 4,032 =
  4 + 3,772 + 256 per head; the French article, second paragraph: the same
  three parts, the older tokens picked by a learned top-k).  Per sequence and KV head: keep
  p < S (sinks), keep p >= L - W (recent window), and among p in [S, L-W)
  keep the k = budget - S - W largest scores; equal scores go to the
  smaller position first.  Everything is kept when L <= budget.

* Prefix top-k thresholds (model card, "Usage" note: the scorer's "prefix
  top-k thresholds").  At decoding step t the tokens p in [S, t - W] have
  left the recent window and compete for the k = budget - S - W scored
  slots.  The threshold of step t is the k-th best of them under the
  keep-set order (higher score first, then smaller position); a token is
  kept at step t iff it ranks at or above the threshold.  With fixed scores
  this is exactly online eviction of the worst token whenever the scored
  slots overflow, and at the last step it gives the keep mask above.

* Static sparse cache (model card, "Cache backends": a cache of fixed size
  whose slots hold the same three shares as the keep mask).  Compaction
  gathers, per sequence and KV head, the kept positions in increasing order
  into fixed slots; a decode step attends one new query per query head over
  the filled slots of its KV head: ``out = sum_s softmax_s(s q.k_s) v_s``.

Readings taken where the pages are silent: the window condition is
``i >= j + W``; the GQA group is summed (not averaged) with consecutive
grouping ``g // G``; the softmax normaliser is the full causal row (sinks
included); the target is the raw mass (no normalisation by the number of
future queries); V is not used; ties in the keep set go to the smaller
position; NaN scores rank below every number.

Inputs may be bf16 bit patterns (uint16 arrays, converted exactly) or float
arrays; the arithmetic is float64 throughout.
"""
from __future__ import annotations

import numpy as np

__all__ = ["as_f64", "row_lse", "future_target", "keep_mask", "prefix_topk_thresholds", "compact_kv",
           "decode_attention", "ROW_BLOCK"]

ROW_BLOCK = 256  # query rows materialised at once


def as_f64(x: np.ndarray) -> np.ndarray:
    """bf16 bits (uint16) -> exact float64; float arrays are widened as they are."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def _sequences(cu_seqlens):
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    return [(int(cu[b]), int(cu[b + 1] - cu[b])) for b in range(len(cu) - 1)]


def _softmax_rows(qg: np.ndarray, kh: np.ndarray, r0: int, r1: int, scale: float):
    """Materialised causal softmax rows r0..r1-1 of one head of one sequence.

    Returns (A, lse) with A[i - r0, j] for j < r1 (entries j > i are 0).
    """
    S = scale * (qg[r0:r1] @ kh[:r1].T)                       # [r1-r0, r1]
    rows = np.arange(r0, r1)[:, None]
    cols = np.arange(r1)[None, :]
    S = np.where(cols <= rows, S, -np.inf)                      # causal mask
    m = S.max(axis=1, keepdims=True)
    P = np.exp(S - m)
    Z = P.sum(axis=1, keepdims=True)
    A = P / Z
    lse = (m + np.log(Z))[:, 0]
    return A, lse


def row_lse(q, k, cu_seqlens, scale: float, rows=None) -> np.ndarray:
    """Natural-log row logsumexp, float64 [H_q, T].

    ``rows`` (optional, sorted int array of global positions) restricts the
    computation to those query rows; other entries are NaN.
    """
    q, k = as_f64(q), as_f64(k)
    T, Hq, _ = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.full((Hq, T), np.nan)
    want = None if rows is None else np.zeros(T, dtype=bool)
    if want is not None:
        want[np.asarray(rows, dtype=np.int64)] = True
    for s, L in _sequences(cu_seqlens):
        for g in range(Hq):
            qg, kh = q[s:s + L, g, :], k[s:s + L, g // G, :]
            for r0 in range(0, L, ROW_BLOCK):
                r1 = min(r0 + ROW_BLOCK, L)
                if want is not None:
                    sel = np.nonzero(want[s + r0:s + r1])[0]
                    for i in sel + r0:                         # one row at a time
                        _, l1 = _softmax_rows(qg, kh, int(i), int(i) + 1, scale)
                        out[g, s + i] = l1[0]
                    continue
                _, lse = _softmax_rows(qg, kh, r0, r1, scale)
                out[g, s + r0:s + r1] = lse
    return out


def future_target(q, k, cu_seqlens, window: int, scale: float, key_lo: int | None = None,
                  return_lse: bool = False, return_far: bool = False):
    """Future-attention target, float64 [H_kv, T].

    ``key_lo`` (optional, a position relative to each sequence's start)
    restricts the work to keys j >= key_lo: only query rows i >= key_lo + W
    are materialised (each in full, so its normaliser is exact); entries of
    keys below key_lo are NaN.

    ``return_lse`` adds the row logsumexp [H_q, T] of the rows materialised;
    ``return_far`` adds ``far[g, i] = sum_{j <= i - W} A_g[i, j]``, the mass
    each query puts on keys at least W back (used by the mass-conservation
    check).
    """
    q, k = as_f64(q), as_f64(k)
    T, Hq, _ = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    W = int(window)
    target = np.zeros((Hkv, T))
    lse_all = np.full((Hq, T), np.nan)
    far = np.full((Hq, T), np.nan)
    for s, L in _sequences(cu_seqlens):
        j_lo = 0 if key_lo is None else max(0, min(int(key_lo), L))
        if key_lo is not None:
            target[:, s:s + j_lo] = np.nan
        i_start = min(L, j_lo + W) if key_lo is not None else 0
        for g in range(Hq):
            h = g // G
            qg, kh = q[s:s + L, g, :], k[s:s + L, h, :]
            for r0 in range(i_start, L, ROW_BLOCK):
                r1 = min(r0 + ROW_BLOCK, L)
                A, lse = _softmax_rows(qg, kh, r0, r1, scale)
                lse_all[g, s + r0:s + r1] = lse
                rows = np.arange(r0, r1)[:, None]
                cols = np.arange(r1)[None, :]
                F = np.where(rows - cols >= W, A, 0.0)         # key has left the window
                far[g, s + r0:s + r1] = F.sum(axis=1)
                col_sum = F.sum(axis=0)                         # mass each key receives
                target[h, s + j_lo:s + r1] += col_sum[j_lo:]
    out = [target]
    if return_lse:
        out.append(lse_all)
    if return_far:
        out.append(far)
    return out[0] if len(out) == 1 else tuple(out)


def keep_mask(score, cu_seqlens, window: int, sinks: int, budgets) -> np.ndarray:
    """Sink + top-k + recent-window keep set, uint8 [H_kv, T] (1 = kept).

    The top-k ranking orders the candidates by (-score, position) with
    NumPy's stable lexsort, which puts NaN scores last.
    """
    score = np.asarray(score)
    Hkv, T = score.shape
    keep = np.zeros((Hkv, T), dtype=np.uint8)
    budgets = np.asarray(budgets, dtype=np.int64)
    W, S = int(window), int(sinks)
    for b, (s, L) in enumerate(_sequences(cu_seqlens)):
        B = int(budgets[b])
        if B < S + W:
            raise ValueError("budget below sinks + window")
        if L <= B:
            keep[:, s:s + L] = 1
            continue
        k_top = B - S - W
        lo, hi = S, L - W                                       # candidate range
        pos = np.arange(lo, hi)
        for h in range(Hkv):
            keep[h, s:s + S] = 1
            keep[h, s + L - W:s + L] = 1
            sc = score[h, s + lo:s + hi].astype(np.float64)
            order = np.lexsort((pos, -sc))                      # -score ascending, then position
            keep[h, s + pos[order[:k_top]]] = 1
    return keep


def prefix_topk_thresholds(score, cu_seqlens, window: int, sinks: int, budgets, steps=None):
    """Per-step eviction thresholds, (thr_score float32 [H_kv, T], thr_pos int32 [H_kv, T]).

    ``steps`` (optional, step indices relative to each sequence's start)
    restricts the work to those steps; other entries are NaN / -2.

    For step t of a sequence (t relative to its start) the candidates are the
    positions p in [S, t - W].  With k = budget - S - W:
      * fewer than k candidates (or none): no eviction yet, thr = (-inf, -1);
      * k = 0 and at least one candidate: nothing is kept, thr = (+inf, -1);
      * otherwise thr = (score, position) of the k-th best candidate in the
        order (-score, position), NaN scores last.
    """
    score = np.asarray(score, dtype=np.float32)
    Hkv, T = score.shape
    thr_s = np.full((Hkv, T), -np.inf, dtype=np.float32)
    thr_p = np.full((Hkv, T), -1, dtype=np.int32)
    budgets = np.asarray(budgets, dtype=np.int64)
    W, S = int(window), int(sinks)
    for b, (s0, L) in enumerate(_sequences(cu_seqlens)):
        k_top = int(budgets[b]) - S - W
        if k_top < 0:
            raise ValueError("budget below sinks + window")
        ts_all = range(L) if steps is None else [int(t) for t in steps if 0 <= int(t) < L]
        if steps is not None:
            thr_s[:, s0:s0 + L] = np.nan
            thr_p[:, s0:s0 + L] = -2
        for h in range(Hkv):
            for t in ts_all:
                thr_s[h, s0 + t], thr_p[h, s0 + t] = -np.inf, -1
                hi = t - W                                     # last candidate position
                if hi < S:
                    continue
                pos = np.arange(S, hi + 1)
                if k_top == 0:
                    thr_s[h, s0 + t] = np.inf
                    continue
                if len(pos) < k_top:
                    continue
                sc = score[h, s0 + S:s0 + hi + 1].astype(np.float64)
                order = np.lexsort((pos, -sc))
                kth = order[k_top - 1]
                thr_s[h, s0 + t] = score[h, s0 + pos[kth]]
                thr_p[h, s0 + t] = pos[kth]
    return thr_s, thr_p


def compact_kv(k, v, keep, cu_seqlens, capacity: int):
    """Gather kept K/V rows into fixed slots.

    Returns (k_cache [B, H_kv, C, d], v_cache [B, H_kv, C, d], pos [B, H_kv, C]
    int32 with -1 in unused slots, count [B, H_kv] int32).  Slots hold the
    kept positions (relative to the sequence start) in increasing order; a row
    with more kept positions than C keeps its first C and reports the full
    count.  K and V keep their input dtype (bf16 bits stay bits).
    """
    k, v, keep = np.asarray(k), np.asarray(v), np.asarray(keep)
    seqs = _sequences(cu_seqlens)
    B, Hkv, d = len(seqs), k.shape[1], k.shape[2]
    kc = np.zeros((B, Hkv, capacity, d), dtype=k.dtype)
    vc = np.zeros((B, Hkv, capacity, d), dtype=v.dtype)
    pos = np.full((B, Hkv, capacity), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv), dtype=np.int32)
    for b, (s0, L) in enumerate(seqs):
        for h in range(Hkv):
            p = np.nonzero(keep[h, s0:s0 + L])[0]
            cnt[b, h] = len(p)
            p = p[:capacity]
            pos[b, h, :len(p)] = p
            kc[b, h, :len(p)] = k[s0 + p, h]
            vc[b, h, :len(p)] = v[s0 + p, h]
    return kc, vc, pos, cnt


def decode_attention(q, k_cache, v_cache, count, scale: float):
    """One decode step over the compacted cache, float64.

    q [B, H_q, d]; k_cache, v_cache [B, H_kv, C, d]; count [B, H_kv].
    Returns (out [B, H_q, d], lse [B, H_q]) with query head g reading KV head
    g // G over its first count[b, g // G] slots.
    """
    q, kc, vc = as_f64(q), as_f64(k_cache), as_f64(v_cache)
    B, Hq, d = q.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        for g in range(Hq):
            h = g // G
            n = int(count[b, h])
            if n == 0:
                continue
            logits = scale * (kc[b, h, :n] @ q[b, g])
            m = logits.max()
            w = np.exp(logits - m)
            Z = w.sum()
            out[b, g] = (w / Z) @ vc[b, h, :n]
            lse[b, g] = m + np.log(Z)
    return out, lse

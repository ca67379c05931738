"""Seeded synthetic inputs for the future-attention-target workloads.

This module only draws random numbers, shapes them and rounds them to bf16.
It holds none of the method's arithmetic (no logits, softmax, targets or
keep sets), so both the CPU oracle's tests and the CUDA path can take their
inputs from it without sharing any of the computation.

The five workloads mirror the shapes the KVpop pages work at: a tiny GQA-2
case, a Qwen3-4B-shaped layer at 4k context, the Qwen3-8B-shaped 16k
distillation layer (KVpop model card, introduction: the model was distilled
with a 16,384-token context and a per-head budget of 4 + 3,772 + 256 = 4,032
entries), a
packed variable-length batch, and a 64k long-context layer.  Q and K are
given post-QK-norm (unit RMS per row), as bf16 bit patterns (uint16).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "get_workload",
    "make_inputs",
    "make_decode_inputs",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "causal_pairs",
    "future_pairs",
    "algorithmic_flops",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: sizes, window/sink/budget and input recipe."""

    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window: int
    sinks: int
    kind: str                       # "gauss" | "heavy" | "topics"
    seqlen: int = 0                 # single-sequence length (0 when varlen)
    budget: int = 0                 # keep budget per KV head (single sequence)
    n_seqs: int = 1                 # varlen: number of packed sequences
    varlen_lo: int = 0              # varlen: inclusive length range
    varlen_hi: int = 0
    keep_ratio: float = 0.0         # varlen: budget_b = floor(ratio * L_b)
    seed: int = 0

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


WORKLOADS = {
    # i.i.d. N(0,1) rows at unit RMS, GQA 2, d=64: budget 128 = 4 + 60 + 64.
    "tiny": Workload("tiny", 2, 1, 64, 64, 4, "gauss", seqlen=512, budget=128),
    # Qwen3-4B-shaped attention layer at 4k: budget 1024 = 4 + 764 + 256.
    "qwen3_4b_4k": Workload("qwen3_4b_4k", 32, 8, 128, 256, 4, "gauss",
                            seqlen=4096, budget=1024),
    # Qwen3-8B-shaped 16k distillation layer with 1% heavy-hitter keys:
    # budget 4032 = 4 + 3772 + 256 (KVpop model card, intro paragraph).
    "qwen3_8b_16k": Workload("qwen3_8b_16k", 32, 8, 128, 256, 4, "heavy",
                             seqlen=16384, budget=4032),
    # 8 packed sequences, lengths uniform in [2048, 16384], keep 25% each.
    "varlen_8x": Workload("varlen_8x", 32, 8, 128, 256, 4, "gauss",
                          n_seqs=8, varlen_lo=2048, varlen_hi=16384,
                          keep_ratio=0.25),
    # 64k context with drifting topics; budget 12.5% of 65536 = 8192.
    "long_64k": Workload("long_64k", 32, 8, 128, 256, 4, "topics",
                         seqlen=65536, budget=8192),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


# ---------------------------------------------------------------- bf16 bits

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _unit_rms(x: np.ndarray) -> np.ndarray:
    """Scale each row (last axis) to unit root-mean-square, in float32."""
    ms = np.mean(np.square(x, dtype=np.float32), axis=-1, keepdims=True, dtype=np.float32)
    return (x / np.sqrt(ms)).astype(np.float32)


# ---------------------------------------------------------------- recipes

def seqlens_of(w: Workload, rng: np.random.Generator | None = None) -> np.ndarray:
    """Sequence lengths; for varlen they are the first draw from the seeded stream."""
    if w.n_seqs == 1 and w.seqlen > 0:
        return np.array([w.seqlen], dtype=np.int64)
    if rng is None:
        rng = np.random.default_rng(w.seed)
    return rng.integers(w.varlen_lo, w.varlen_hi, size=w.n_seqs, endpoint=True).astype(np.int64)


def budgets_of(w: Workload, seqlens: np.ndarray) -> np.ndarray:
    if w.keep_ratio > 0:
        return np.floor(w.keep_ratio * seqlens.astype(np.float64)).astype(np.int32)
    return np.full(len(seqlens), w.budget, dtype=np.int32)


def _gauss_qk(rng, T, w):
    q = rng.standard_normal((T, w.n_q_heads, w.head_dim), dtype=np.float32)
    k = rng.standard_normal((T, w.n_kv_heads, w.head_dim), dtype=np.float32)
    return _unit_rms(q), _unit_rms(k)


def _plant_heavy_hitters(rng, q, k, seqlens, w, fraction=0.01, gain=3.0):
    """Replace 1% of keys per KV head by gain * (unit-RMS mean query direction) + N(0,1) noise.

    The mean direction is taken over the positions and the query heads of the
    KV head's group; the planted key is not re-normalised, so it really is
    about `gain` times larger along that direction.
    """
    G = w.group
    starts = np.concatenate([[0], np.cumsum(seqlens)])
    for b, L in enumerate(seqlens):
        s = int(starts[b])
        n_heavy = int(round(fraction * int(L)))
        for h in range(w.n_kv_heads):
            qg = q[s:s + L, h * G:(h + 1) * G, :]
            u = qg.reshape(-1, w.head_dim).mean(axis=0, dtype=np.float64).astype(np.float32)
            u = _unit_rms(u[None, :])[0]
            idx = rng.choice(int(L), size=n_heavy, replace=False)
            noise = rng.standard_normal((n_heavy, w.head_dim), dtype=np.float32)
            k[s + idx, h, :] = gain * u[None, :] + noise
    return q, k


def _drifting_topics(rng, seqlens, w, n_centres=16, segment=4096, past_weight=0.5):
    """Keys around 16 per-KV-head centres that switch every 4096 positions.

    Segment t uses centre pi(t) (pi a seeded permutation, cycled when there
    are more segments than centres).  Queries mix the current centre with
    0.5 x the centre of one seeded earlier segment t' < t (none for t = 0).
    """
    T = int(np.sum(seqlens))
    d, G = w.head_dim, w.group
    centres = _unit_rms(rng.standard_normal((w.n_kv_heads, n_centres, d), dtype=np.float32))
    perm = rng.permutation(n_centres)
    q = np.empty((T, w.n_q_heads, d), dtype=np.float32)
    k = np.empty((T, w.n_kv_heads, d), dtype=np.float32)
    starts = np.concatenate([[0], np.cumsum(seqlens)])
    for b, L in enumerate(seqlens):
        s, L = int(starts[b]), int(L)
        n_seg = (L + segment - 1) // segment
        past = [None] + [int(rng.integers(0, t)) for t in range(1, n_seg)]
        for t in range(n_seg):
            p0, p1 = s + t * segment, s + min((t + 1) * segment, L)
            n = p1 - p0
            cur = perm[t % n_centres]
            ck = centres[:, cur, :]                                      # [Hkv, d]
            k[p0:p1] = ck[None] + rng.standard_normal((n, w.n_kv_heads, d), dtype=np.float32)
            cq = np.repeat(ck, G, axis=0)                                # [Hq, d]
            if past[t] is not None:
                cq = cq + past_weight * np.repeat(centres[:, perm[past[t] % n_centres], :], G, axis=0)
            q[p0:p1] = cq[None] + rng.standard_normal((n, w.n_q_heads, d), dtype=np.float32)
    return _unit_rms(q), _unit_rms(k)


def make_inputs(w: Workload | str, seed: int | None = None) -> dict:
    """Draw one workload's inputs.

    Returns a dict with
      q_bits   uint16 [T, H_q, d]   bf16 bit patterns
      k_bits   uint16 [T, H_kv, d]
      cu_seqlens int32 [B+1]
      budgets  int32 [B]            keep budget per sequence (per KV head)
    plus the workload's scalars (window, sinks, scale, ...).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if seed is not None:
        w = dataclasses.replace(w, seed=seed)
    rng = np.random.default_rng(w.seed)
    seqlens = seqlens_of(w, rng)
    T = int(seqlens.sum())
    if w.kind == "gauss":
        q, k = _gauss_qk(rng, T, w)
    elif w.kind == "heavy":
        q, k = _gauss_qk(rng, T, w)
        q, k = _plant_heavy_hitters(rng, q, k, seqlens, w)
    elif w.kind == "topics":
        q, k = _drifting_topics(rng, seqlens, w)
    else:
        raise ValueError(f"unknown input kind {w.kind!r}")
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    return {
        "workload": w,
        "q_bits": f32_to_bf16_bits(q),
        "k_bits": f32_to_bf16_bits(k),
        "cu_seqlens": cu,
        "budgets": budgets_of(w, seqlens),
        "window": w.window,
        "sinks": w.sinks,
        "scale": 1.0 / math.sqrt(w.head_dim),
    }


def make_decode_inputs(w: Workload | str, seed: int | None = None) -> dict:
    """Values for the static cache and one decode query per sequence.

    V rows are i.i.d. N(0,1) (bf16 bits, [T, H_kv, d]); the decode query is a
    unit-RMS N(0,1) row per query head ([B, H_q, d]).  Drawn from a stream of
    their own (seed + 1000), so the Q/K inputs stay unchanged.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    s = w.seed if seed is None else seed
    seqlens = seqlens_of(w, np.random.default_rng(s))
    rng = np.random.default_rng(s + 1000)
    T = int(seqlens.sum())
    v = rng.standard_normal((T, w.n_kv_heads, w.head_dim), dtype=np.float32)
    q_dec = _unit_rms(rng.standard_normal((len(seqlens), w.n_q_heads, w.head_dim), dtype=np.float32))
    return {"v_bits": f32_to_bf16_bits(v), "q_dec_bits": f32_to_bf16_bits(q_dec)}


def random_qk(T: int, n_q_heads: int, n_kv_heads: int, head_dim: int, seed: int,
              q_zero: bool = False, k_zero: bool = False, gain: float = 1.0) -> tuple:
    """Plain i.i.d. unit-RMS Q/K bits for ad-hoc shapes (edge-case tests)."""
    rng = np.random.default_rng(seed)
    q = _unit_rms(rng.standard_normal((T, n_q_heads, head_dim), dtype=np.float32)) * np.float32(gain)
    k = _unit_rms(rng.standard_normal((T, n_kv_heads, head_dim), dtype=np.float32)) * np.float32(gain)
    if q_zero:
        q[:] = 0
    if k_zero:
        k[:] = 0
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k)


# ---------------------------------------------------------------- counts

def causal_pairs(seqlens) -> int:
    """Pairs (i, j) with j <= i inside each sequence (row-logsumexp pass)."""
    return int(sum(int(L) * (int(L) + 1) // 2 for L in seqlens))


def future_pairs(seqlens, window: int) -> int:
    """Pairs (i, j) with i >= j + W inside each sequence (transposed pass)."""
    tot = 0
    for L in seqlens:
        n = max(int(L) - window, 0)
        tot += n * (n + 1) // 2
    return tot


def algorithmic_flops(seqlens, n_q_heads: int, head_dim: int, window: int) -> dict:
    """Tensor flops of both passes, counting only unmasked (i, j) pairs: 2 d per pair per head."""
    n_lse = causal_pairs(seqlens)
    n_tgt = future_pairs(seqlens, window)
    per = 2 * head_dim * n_q_heads
    return {"lse": per * n_lse, "target": per * n_tgt, "total": per * (n_lse + n_tgt),
            "pairs_lse": n_lse * n_q_heads, "pairs_target": n_tgt * n_q_heads}

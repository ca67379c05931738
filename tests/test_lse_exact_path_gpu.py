"""Row logsumexp's exact path on inputs whose scores leave the fp32 range of the fast path.

Pass 1 sums a row's first key tile at offset 0 and keeps the running offset
while every tile's sum stays in [2^-64, 2^64).  A tile outside that range
(an overflowing or vanishing sum) takes the exact max of its scores, which the
kernel recomputes on CUDA cores from Q and K (the tile's accumulator has
already gone back to the tensor cores by then).  Ordinary inputs never reach
that path; these do:

- large-gain i.i.d. Q and K (score standard deviation 36, i.e. ~52 in log2
  units): most first tiles overflow;
- a shared direction u (entries +-1) with q = 8 u and k = -c u on the first
  256 keys, +c u after them (c = 1..8 per key): every first tile sums to
  exactly 0 at offset 0 (scores near -724) and the later tiles jump by more
  than 2^128 over the running offset.  All scores are exact integers times
  the scale, so the oracle's fp64 values are exact.

Each case runs the whole hot path and compares lse, targets and the keep mask
with the fp64 oracle (the same bounds as the parity tests).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import _binding as B
from future_attention_targets_b200.workloads import f32_to_bf16_bits, random_qk

pytestmark = pytest.mark.gpu

TARGET_TOL, LSE_TOL = 2e-3, 2e-4


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def check(q_bits, k_bits, seqlens, W, S):
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    d = q_bits.shape[2]
    scale = 1.0 / math.sqrt(d)
    budgets = [min(int(L), W + S + 37) for L in seqlens]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse, tgt, keep = B.future_targets(dev(q_bits), dev(k_bits), cu, W, S, budgets, scale=scale, status=st)
    B.check_status(st)
    ref_t, ref_l = oracle.future_target(q_bits, k_bits, cu, W, scale, return_lse=True)
    lse_h = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(lse_h))
    err_l = float(np.max(np.abs(lse_h - ref_l), initial=0.0))
    assert err_l <= LSE_TOL, f"lse error {err_l:.3e}"
    tgt_h = tgt.cpu().numpy()
    err_t = float(np.max(np.abs(tgt_h.astype(np.float64) - ref_t) / np.maximum(np.abs(ref_t), 1e-3), initial=0.0))
    assert err_t <= TARGET_TOL, f"target error {err_t:.3e}"
    np.testing.assert_array_equal(keep.cpu().numpy(), oracle.keep_mask(tgt_h, cu, W, S, budgets))
    return err_l, err_t


@pytest.mark.parametrize("d", [128, 64])
def test_large_gain_scores(d):
    seqlens = (700, 300)
    q_bits, k_bits = random_qk(sum(seqlens), 4, 2, d, seed=91 + d, gain=6.0)
    check(q_bits, k_bits, seqlens, 16, 4)


@pytest.mark.parametrize("d", [128, 64])
def test_vanishing_first_tiles_and_jumps(d):
    seqlens = (900, 260)
    T, hq, hkv = sum(seqlens), 4, 2
    rng = np.random.default_rng(7 + d)
    u = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=d)
    q = np.broadcast_to(8.0 * u, (T, hq, d)).astype(np.float32)
    k = np.empty((T, hkv, d), dtype=np.float32)
    start = 0
    for L in seqlens:
        c = rng.integers(1, 9, size=(L, hkv)).astype(np.float32)
        sign = np.where(np.arange(L) < 256, -1.0, 1.0).astype(np.float32)
        k[start:start + L] = (sign[:, None] * c)[:, :, None] * u[None, None, :]
        start += L
    check(f32_to_bf16_bits(q), f32_to_bf16_bits(k), seqlens, 0, 2)

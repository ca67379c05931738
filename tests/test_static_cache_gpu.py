"""Static fixed-budget cache on the GPU against the CPU oracle: compaction of
the kept K/V rows (exact) and one decode step of attention over them
(elementwise |gpu - oracle| <= 2e-3 * max(|oracle|, 1e-3))."""
import math

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import compact_kv, decode_attention, future_targets, keep_mask
from future_attention_targets_b200.workloads import make_decode_inputs, make_inputs, random_qk

pytestmark = pytest.mark.gpu
TOL = 2e-3


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def rel_err(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.max(np.abs(g - o) / np.maximum(np.abs(o), 1e-3))) if g.size else 0.0


def check_compaction(k_bits, v_bits, keep, cu, C):
    kc, vc, pos, cnt = compact_kv(dev(k_bits), dev(v_bits), torch.from_numpy(keep).cuda(), cu, C)
    rk, rv, rp, rc = oracle.compact_kv(k_bits, v_bits, keep, cu, C)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)
    np.testing.assert_array_equal(pos.cpu().numpy(), rp)
    np.testing.assert_array_equal(kc.cpu().view(torch.int16).numpy().view(np.uint16), rk)
    np.testing.assert_array_equal(vc.cpu().view(torch.int16).numpy().view(np.uint16), rv)
    return kc, vc, cnt, (rk, rv, rc)


@pytest.mark.parametrize("seqlens,Hkv,d,C,p", [
    ((700,), 2, 128, 300, 0.3),
    ((1,), 1, 64, 4, 1.0),
    ((1300, 0, 37, 2500), 3, 64, 900, 0.35),        # empty sequence, rows over capacity (truncated)
    ((5000,), 2, 128, 5000, 1.0),                   # everything kept
])
def test_compaction_random_masks(seqlens, Hkv, d, C, p):
    T = sum(seqlens)
    rng = np.random.default_rng(T)
    k_bits, _ = random_qk(T, Hkv, Hkv, d, seed=T)
    v_bits, _ = random_qk(T, Hkv, Hkv, d, seed=T + 1)
    keep = (rng.random((Hkv, T)) < p).astype(np.uint8)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    check_compaction(k_bits, v_bits, keep, cu, C)


@pytest.mark.parametrize("seqlens,C", [((16384,), 4032), ((3001, 17, 5000), 1000), ((70000,), 129)])
def test_compaction_clustered_masks(seqlens, C):
    """Kept positions packed at the front (as large targets of early keys give) and
    unaligned sequence starts: the slot-range CTAs must still find every row."""
    T, Hkv, d = sum(seqlens), 2, 128
    k_bits, _ = random_qk(T, Hkv, Hkv, d, seed=5)
    v_bits, _ = random_qk(T, Hkv, Hkv, d, seed=6)
    keep = np.zeros((Hkv, T), dtype=np.uint8)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    rng = np.random.default_rng(9)
    for b, L in enumerate(seqlens):
        s0 = cu[b]
        keep[0, s0:s0 + min(L, 3 * C // 4)] = 1                        # a dense front block
        keep[0, s0 + max(0, L - 256):s0 + L] = 1                       # and the recent window
        keep[1, s0:s0 + L] = rng.random(L) < (C / max(L, 1)) * np.linspace(2, 0, L)   # density falling with p
    check_compaction(k_bits, v_bits, keep, cu, C)


@pytest.mark.parametrize("G,d,C,fill", [(4, 128, 1000, [1000, 3, 0, 517]), (2, 64, 300, [300, 1, 299, 0]),
                                        (1, 128, 40, [40, 40, 7, 1]), (16, 128, 600, [600, 256, 257, 255]),
                                        (8, 64, 513, [513, 512, 1, 2]),
                                        # warp (32-slot) and CTA (128-slot) boundaries, several sequences
                                        (4, 128, 300, [[129, 32, 33, 95], [1, 300, 128, 31], [0, 0, 0, 64]]),
                                        (2, 64, 130, [[127, 128], [129, 130]]),
                                        # the merge stages up to 64 splits in shared memory, streams beyond
                                        (4, 128, 8192, [8192, 8191, 1, 0]),
                                        (2, 64, 9000, [9000, 8193, 4, 0])])
def test_decode_attention_random_cache(G, d, C, fill):
    fill = fill if isinstance(fill[0], list) else [fill]
    B, Hkv = len(fill), len(fill[0])
    rng = np.random.default_rng(C + G)
    kc = rng.standard_normal((B, Hkv, C, d)).astype(np.float32) * 2.0
    vc = rng.standard_normal((B, Hkv, C, d)).astype(np.float32)
    q = rng.standard_normal((B, Hkv * G, d)).astype(np.float32)
    from future_attention_targets_b200.workloads import f32_to_bf16_bits
    kb, vb, qb = f32_to_bf16_bits(kc), f32_to_bf16_bits(vc), f32_to_bf16_bits(q)
    cnt = np.array(fill, dtype=np.int32)
    scale = 1.0 / math.sqrt(d)
    out, lse = decode_attention(dev(qb), dev(kb), dev(vb), torch.from_numpy(cnt).cuda(), scale)
    ro, rl = oracle.decode_attention(qb, kb, vb, cnt, scale)
    assert rel_err(out.cpu().numpy(), ro) <= TOL
    lse_g = lse.cpu().numpy()
    empty = ~np.isfinite(rl)
    assert np.all(np.isneginf(lse_g[empty])) and np.all(out.cpu().numpy()[np.repeat(cnt == 0, G, axis=1)] == 0)
    assert np.max(np.abs(lse_g[~empty] - rl[~empty])) <= 1e-4


@pytest.mark.parametrize("name", ["qwen3_4b_4k", "varlen_8x"])
def test_end_to_end_static_cache(name):
    """targets -> keep mask -> compaction -> one decode step, on a full workload."""
    d = make_inputs(name)
    w = d["workload"]
    dd = make_decode_inputs(name)
    _, tgt, keep = future_targets(dev(d["q_bits"]), dev(d["k_bits"]), d["cu_seqlens"], d["window"], d["sinks"],
                                  d["budgets"], scale=d["scale"])
    keep_np = keep.cpu().numpy()
    C = int(max(d["budgets"]))
    kc, vc, cnt, (rk, rv, rc) = check_compaction(d["k_bits"], dd["v_bits"], keep_np, d["cu_seqlens"], C)
    assert np.all(rc == np.minimum(np.asarray(d["budgets"])[:, None], np.diff(d["cu_seqlens"])[:, None]))
    out, lse = decode_attention(dev(dd["q_dec_bits"]), kc, vc, cnt, d["scale"])
    ro, rl = oracle.decode_attention(dd["q_dec_bits"], rk, rv, rc, d["scale"])
    assert rel_err(out.cpu().numpy(), ro) <= TOL
    assert np.max(np.abs(lse.cpu().numpy() - rl)) <= 1e-4

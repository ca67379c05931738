"""The bounds-checking debug build (libkvpop_debug.so) on the GPU, through the C ABI.

The same sources compiled with KVPOP_DEBUG make every kernel check the index
of each data-dependent global or shared-memory access before making it; a
failed check skips the access and records a code in a device word registered
with kvpop_debug_set_word (nothing traps).  Here every entry point runs under
that build on the tiny workload, the edge shapes of the parity tests and the
512-sequence ragged batch: the word must stay 0 and the results must still
match the fp64 oracle.  The self-test kernel's check, which fails by design
(its guarded store is skipped), must land its code in the word, which shows
that a failing check is recorded.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from future_attention_targets_b200 import _binding as B
from future_attention_targets_b200.build import build
from future_attention_targets_b200.workloads import make_inputs, random_qk
from test_parity_gpu import EDGE

pytestmark = pytest.mark.gpu

TARGET_TOL, LSE_TOL = 2e-3, 2e-4   # lse: as in test_parity_gpu


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def rel_err(gpu, ref):
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-3), initial=0.0))


def glob_err(gpu, ref):
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(gpu - ref), initial=0.0) / max(float(np.max(np.abs(ref), initial=0.0)), 1e-3))


@pytest.fixture(scope="module")
def word():
    """Switches the binding to the debug build for this module, with a registered, zero-filled word."""
    old = B.use_library(build(debug=True))
    w = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.debug_set_word(w)
    try:
        yield w
    finally:
        B.debug_set_word(None)
        B.use_library(old)


def assert_clean(word):
    torch.cuda.synchronize()
    code = int(word.item())
    assert code == 0, f"bounds check failed: kernel {(code >> 16) & 0xff}, site {(code >> 8) & 0xff}"


def test_selftest_check_is_recorded(word):
    own = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.debug_selftest(own)
    torch.cuda.synchronize()
    assert int(own.item()) == B.BOUNDS | (1 << 8) | (10 << 16)
    with pytest.raises(B.KvpopError, match="BOUNDS"):
        B.check_status(own)
    assert_clean(word)


def all_entry_points(q_bits, k_bits, cu, W, S, budgets, scale, word, v_seed):
    """Every entry point on one problem; results against the oracle; the debug word after each group."""
    q, k = dev(q_bits), dev(k_bits)
    hq, hkv, d = q.shape[1], k.shape[1], q.shape[2]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse, tgt, keep = B.future_targets(q, k, cu, W, S, budgets, scale=scale, status=st)
    B.check_status(st)
    assert_clean(word)
    ref_t, ref_l = oracle.future_target(q_bits, k_bits, cu, W, scale, return_lse=True)
    tgt_h = tgt.cpu().numpy()
    assert rel_err(tgt_h, ref_t) <= TARGET_TOL
    assert float(np.max(np.abs(lse.cpu().numpy() - ref_l), initial=0.0)) <= LSE_TOL
    np.testing.assert_array_equal(keep.cpu().numpy(), oracle.keep_mask(tgt_h, cu, W, S, budgets))

    # The standalone passes (normaliser rows from lse), the split pass and the single launch.
    l2 = B.row_lse(q, k, cu, scale, status=st)
    t2 = B.future_target(q, k, cu, W, l2, scale, status=st)
    t3 = B.future_target_split(q, k, cu, W, l2, scale, status=st)
    fused = B.future_targets_fused(q, k, cu, W, S, budgets, scale=scale, status=st)
    B.check_status(st)
    assert_clean(word)
    for t in (t2, t3, fused[1]):
        assert rel_err(t.cpu().numpy(), ref_t) <= TARGET_TOL

    # Host buffers in and out.
    pipe = B.HostPipeline(cu, hq, hkv, d, W, S, budgets, scale=scale)
    t_h, _ = pipe(torch.from_numpy(q_bits.view(np.int16)).view(torch.bfloat16).pin_memory(),
                  torch.from_numpy(k_bits.view(np.int16)).view(torch.bfloat16).pin_memory())
    B.check_status(pipe.status)
    assert_clean(word)
    assert torch.equal(t_h, tgt.cpu())

    # Thresholds, compaction and decode (workspace and allocation-free forms).
    ts, tp = B.prefix_topk_thresholds(tgt, cu, W, S, budgets)
    assert_clean(word)
    rs, rp = oracle.prefix_topk_thresholds(tgt_h, cu, W, S, budgets)
    np.testing.assert_array_equal(tp.cpu().numpy(), rp)
    np.testing.assert_array_equal(ts.cpu().numpy(), rs)
    C = max(int(max(budgets)), 1)
    v_bits, _ = random_qk(q.shape[0], hkv, hkv, d, seed=v_seed)
    kc, vc, pos, cnt = B.compact_kv(k, dev(v_bits), keep, cu, C)
    assert_clean(word)
    rk, rv, rpos, rc = oracle.compact_kv(k_bits, v_bits, keep.cpu().numpy(), cu, C)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rc)
    np.testing.assert_array_equal(pos.cpu().numpy(), rpos)
    nb = len(cu) - 1
    if hq // hkv <= 16 and (hq // hkv) & (hq // hkv - 1) == 0 and nb <= 512:
        qd_bits, _ = random_qk(nb, hq, hkv, d, seed=v_seed + 1)
        qd = dev(qd_bits.reshape(nb, hq, d))
        out, dl = B.decode_attention(qd, kc, vc, cnt, scale)
        assert_clean(word)
        ro, rl = oracle.decode_attention(qd_bits.reshape(nb, hq, d), rk, rv, rc, scale)
        # Outputs are weighted means of unit-variance values, some near zero: the global reading of the
        # tolerance (this file checks bounds; test_static_cache_gpu holds the decode step's own bar).
        assert glob_err(out.cpu().numpy(), ro) <= TARGET_TOL
        shape = B.CacheShape(nb, hq, hkv, d, C)
        if B.lib().kvpop_decode_workspace_bytes(shape) <= (4 << 20):
            o2 = torch.empty_like(out)
            l2n = torch.empty_like(dl)
            assert B.lib().kvpop_decode_attention_noalloc(qd.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                                          cnt.data_ptr(), shape, scale, o2.data_ptr(),
                                                          l2n.data_ptr(), None) == B.OK
            assert_clean(word)
            assert glob_err(o2.cpu().numpy(), ro) <= TARGET_TOL


def test_tiny_workload(word):
    d = make_inputs("tiny")
    all_entry_points(d["q_bits"], d["k_bits"], d["cu_seqlens"], d["window"], d["sinks"], d["budgets"], d["scale"],
                     word, 31)


@pytest.mark.parametrize("case", EDGE, ids=[f"L{c[0]}-G{c[1] // c[2]}-d{c[3]}-W{c[4]}" for c in EDGE])
def test_edge_shapes(word, case):
    seqlens, hq, hkv, d, W, gain = case
    T = sum(seqlens)
    q_bits, k_bits = random_qk(T, hq, hkv, d, seed=T + W, gain=gain)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    budgets = [W + 4 + 7] * len(seqlens)
    all_entry_points(q_bits, k_bits, cu, W, 4, budgets, 1.0 / math.sqrt(d), word, T + 1)


def test_max_batch(word):
    rng = np.random.default_rng(21)
    seqlens = rng.integers(0, 300, 512)
    seqlens[:6] = [0, 1, 16, 17, 0, 299]
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    q_bits, k_bits = random_qk(int(cu[-1]), 4, 2, 64, seed=22, gain=2.0)
    budgets = [max(2 + 16, int(L) // 2) for L in seqlens]
    all_entry_points(q_bits, k_bits, cu, 16, 2, budgets, 1.0 / 8.0, word, 23)


def test_large_scores_exact_path(word):
    """Scores large enough that pass 1 takes its exact path (scores recomputed from Q and K on CUDA
    cores) for most rows: every index that path reads is checked too."""
    seqlens = (700, 300)
    q_bits, k_bits = random_qk(sum(seqlens), 4, 2, 128, seed=219, gain=6.0)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    all_entry_points(q_bits, k_bits, cu, 16, 4, [16 + 4 + 37] * len(seqlens), 1.0 / math.sqrt(128), word, 220)

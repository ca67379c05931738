"""Seeded input generators: determinism, bf16 rounding, shapes and recipes."""
import numpy as np
import pytest
import torch

from future_attention_targets_b200.workloads import (
    WORKLOADS, algorithmic_flops, bf16_bits_to_f32, causal_pairs, f32_to_bf16_bits,
    future_pairs, make_inputs)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 65504.0, 3.0e38], dtype=np.float32)])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(f32_to_bf16_bits(x), ref)
    back = bf16_bits_to_f32(ref)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("name", ["tiny", "qwen3_4b_4k"])
def test_deterministic_and_unit_rms(name):
    a, b = make_inputs(name), make_inputs(name)
    np.testing.assert_array_equal(a["q_bits"], b["q_bits"])
    np.testing.assert_array_equal(a["k_bits"], b["k_bits"])
    w = WORKLOADS[name]
    q = bf16_bits_to_f32(a["q_bits"]).astype(np.float64)
    rms = np.sqrt((q ** 2).mean(axis=-1))
    assert np.allclose(rms, 1.0, atol=1e-2)
    assert a["q_bits"].shape == (w.seqlen, w.n_q_heads, w.head_dim)
    assert a["k_bits"].shape == (w.seqlen, w.n_kv_heads, w.head_dim)
    assert list(a["cu_seqlens"]) == [0, w.seqlen]
    assert list(a["budgets"]) == [w.budget]
    c = make_inputs(name, seed=1)
    assert not np.array_equal(a["q_bits"], c["q_bits"])


def test_heavy_hitters_planted():
    d = make_inputs("qwen3_8b_16k")
    k = bf16_bits_to_f32(d["k_bits"]).astype(np.float64)
    norms = np.sqrt((k ** 2).mean(axis=-1))                   # unit RMS = 1, heavy ~ sqrt(10)
    heavy = norms > 2.0
    assert np.all(heavy.sum(axis=0) == round(0.01 * 16384))


def test_varlen_lengths_and_budgets():
    d = make_inputs("varlen_8x")
    L = np.diff(d["cu_seqlens"])
    assert len(L) == 8 and L.min() >= 2048 and L.max() <= 16384
    np.testing.assert_array_equal(d["budgets"], np.floor(0.25 * L).astype(np.int32))
    assert np.all(d["budgets"] >= 4 + 256)


def test_pair_and_flop_counts():
    # brute-force counts on small lengths
    for Ls, W in [((5, 9), 0), ((5, 9), 3), ((17,), 20)]:
        n1 = sum(1 for L in Ls for i in range(L) for j in range(i + 1))
        n2 = sum(1 for L in Ls for i in range(L) for j in range(i + 1) if i - j >= W)
        assert causal_pairs(Ls) == n1 and future_pairs(Ls, W) == n2
    f = algorithmic_flops([16384], 32, 128, 256)
    assert abs(f["total"] - 2.165e12) / 2.165e12 < 2e-3

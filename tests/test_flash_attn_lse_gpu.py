"""Cross-check of the row logsumexp against an independent implementation.

flash_attn's causal varlen forward returns the natural-log softmax normaliser
of every (query head, row), the quantity kvpop_row_lse computes.  This test
compares the two on every row at full size, including the 16k workload where
the oracle checks only sampled rows (the oracle stays the reference for
parity; this is a second, unrelated implementation).  Skipped when flash_attn
is not importable.
"""
import math

import numpy as np
import pytest
import torch

from future_attention_targets_b200 import row_lse
from future_attention_targets_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu
flash_attn = pytest.importorskip("flash_attn")

LSE_TOL = 2e-4   # the row logsumexp's own bound (see test_parity_gpu)


@pytest.mark.parametrize("name", ["qwen3_4b_4k", "qwen3_8b_16k", "varlen_8x"])
def test_row_lse_matches_flash_attn(name):
    from flash_attn import flash_attn_varlen_func
    d = make_inputs(name)
    q = torch.from_numpy(d["q_bits"].view(np.int16)).view(torch.bfloat16).cuda()
    k = torch.from_numpy(d["k_bits"].view(np.int16)).view(torch.bfloat16).cuda()
    cu = d["cu_seqlens"]
    cu_t = torch.from_numpy(np.asarray(cu, dtype=np.int32)).cuda()
    max_len = int(np.max(np.diff(cu)))
    _, lse_fa, _ = flash_attn_varlen_func(q, k, torch.zeros_like(k), cu_t, cu_t, max_len, max_len,
                                          softmax_scale=d["scale"], causal=True, return_attn_probs=True)
    ours = row_lse(q, k, cu, d["scale"])
    assert tuple(lse_fa.shape) == tuple(ours.shape)
    assert float((lse_fa.float() - ours).abs().max()) <= LSE_TOL

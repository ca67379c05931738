"""Every target of the full-size workloads against a plain PyTorch fp32 computation on the GPU.

The oracle checks the full-size workloads on sampled keys (it would need the
whole causal softmax for the others).  This test recomputes ALL targets with
ordinary PyTorch fp32 operations (cuBLAS matmul with TF32 off, logsumexp,
exp, column sums over rows of 2048 queries at a time) and compares every key
with the kernels' targets under the same elementwise tolerance.  It is a
second, unrelated implementation, not the parity reference; its own error
(fp32 dot products and exponentials) is about 1e-5 relative.
"""
import numpy as np
import pytest
import torch

from future_attention_targets_b200 import future_targets
from future_attention_targets_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu
TARGET_TOL = 2e-3
ROWS = 2048


def torch_targets(q, k, cu, W, scale):
    """target [H_kv, T] in fp32 from q [T, H_q, d], k [T, H_kv, d] (bf16 CUDA tensors)."""
    T, Hq, _ = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = torch.zeros((Hkv, T), dtype=torch.float32, device=q.device)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        L = s1 - s0
        for g in range(Hq):
            h = g // G
            kf = k[s0:s1, h].float()
            for r0 in range(0, L, ROWS):
                r1 = min(L, r0 + ROWS)
                S = (q[s0 + r0:s0 + r1, g].float() @ kf[:r1].T) * scale           # rows r0..r1, keys 0..r1
                i = torch.arange(r0, r1, device=q.device)[:, None]
                j = torch.arange(r1, device=q.device)[None, :]
                S = S.masked_fill(j > i, float("-inf"))
                P = torch.exp(S - torch.logsumexp(S, dim=1, keepdim=True))
                P = P.masked_fill(j > i - W, 0.0)                                 # only keys with i >= j + W
                out[h, s0:s0 + r1] += P.sum(dim=0)
    return out


@pytest.mark.parametrize("name", ["qwen3_8b_16k", "varlen_8x", "long_64k"])
def test_all_targets_against_torch_fp32(name):
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        d = make_inputs(name)
        q = torch.from_numpy(d["q_bits"].view(np.int16)).view(torch.bfloat16).cuda()
        k = torch.from_numpy(d["k_bits"].view(np.int16)).view(torch.bfloat16).cuda()
        cu, W = d["cu_seqlens"], d["window"]
        _, tgt, _ = future_targets(q, k, cu, W, d["sinks"], d["budgets"], scale=d["scale"])
        ref = torch_targets(q, k, cu, W, d["scale"])
        rel = ((tgt.double() - ref.double()).abs() / ref.double().abs().clamp_min(1e-3)).max().item()
        assert rel <= TARGET_TOL, rel
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev

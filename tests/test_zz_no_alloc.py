"""The allocation-free decode step (kvpop_decode_attention_noalloc) against
the workspace version (kvpop_decode_attention), both called through the C ABI.

Some callers may not allocate device memory while they run a decode step
(memory owned by another framework's allocator or a pre-reserved pool, decode
loops that cannot afford cudaMalloc's synchronisation, plugin hooks without a
scratch buffer); the allocation-free entry point keeps its split partials in
a fixed array inside the library instead.  Two calls in a row must both agree
with the workspace version, and the test must hold in a fresh process as well
as after the other GPU tests (this file is collected last on purpose).
"""
import math

import numpy as np
import pytest
import torch

from future_attention_targets_b200 import _binding as B
from future_attention_targets_b200.workloads import f32_to_bf16_bits

pytestmark = pytest.mark.gpu
TOL = 2e-3     # the decode-attention tolerance used by the other GPU tests


def _rel_err(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.max(np.abs(g - o) / np.maximum(np.abs(o), 1e-3)))


def test_noalloc_decode_matches_workspace_version_twice():
    lib = B.lib()
    Bn, Hkv, G, d, C = 2, 8, 4, 128, 4032
    rng = np.random.default_rng(2024)
    to_dev = lambda a: torch.from_numpy(f32_to_bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
    kc = to_dev(rng.standard_normal((Bn, Hkv, C, d)).astype(np.float32))
    vc = to_dev(rng.standard_normal((Bn, Hkv, C, d)).astype(np.float32))
    q = to_dev(rng.standard_normal((Bn, Hkv * G, d)).astype(np.float32))
    count = torch.from_numpy(rng.integers(0, C + 1, size=(Bn, Hkv)).astype(np.int32)).cuda()
    shape = B.CacheShape(Bn, Hkv * G, Hkv, d, C)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream().cuda_stream

    ws = torch.empty(lib.kvpop_decode_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    ref_out = torch.empty((Bn, Hkv * G, d), dtype=torch.float32, device="cuda")
    ref_lse = torch.empty((Bn, Hkv * G), dtype=torch.float32, device="cuda")
    st = lib.kvpop_decode_attention(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), count.data_ptr(), shape, scale,
                                    ref_out.data_ptr(), ref_lse.data_ptr(), ws.data_ptr(), ws.numel(), stream)
    assert st == B.OK, lib.kvpop_last_error()

    for call in range(2):
        out = torch.full((Bn, Hkv * G, d), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((Bn, Hkv * G), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.kvpop_decode_attention_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), count.data_ptr(),
                                                shape, scale, out.data_ptr(), lse.data_ptr(), stream)
        assert st == B.OK, lib.kvpop_last_error()
        torch.cuda.synchronize()
        assert _rel_err(out.cpu().numpy(), ref_out.cpu().numpy()) <= TOL, f"call {call}"
        finite = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(lse), finite), f"call {call}"
        assert float((lse[finite] - ref_lse[finite]).abs().max()) <= 1e-4, f"call {call}"

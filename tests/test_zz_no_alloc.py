"""The allocation-free decode step (kvpop_decode_attention_noalloc) through the C ABI.

Some callers may not allocate device memory while they run a decode step:
code whose device memory all belongs to another framework's allocator or a
pre-reserved pool, decode loops that cannot afford cudaMalloc's
synchronisation, plugin hooks that are handed no scratch buffer.  For them
the allocation-free entry point keeps its split partials in a fixed array
inside the library.  These tests check that
  * two calls in a row both agree with the workspace version
    (kvpop_decode_attention) and with the fp64 oracle's decode step;
  * the calls leave the device's free memory unchanged (nothing allocated);
  * a smaller shape after a larger one is still correct, although the shared
    array keeps the larger call's partials;
  * all of it holds in a fresh process, where the first call on the device
    looks up the array's address (run as a subprocess of this file), as well
    as after the other GPU tests (this file is collected last on purpose).
"""
import math
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

TOL = 2e-3       # elementwise relative bound on the decode output (floor 1e-3), as in the other decode tests
LSE_TOL = 1e-4   # absolute bound on its natural-log lse
SCRATCH = 4 << 20  # the fixed array's size stated in include/kvpop.h


def _rel_err(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.max(np.abs(g - o) / np.maximum(np.abs(o), 1e-3)))


def _case(Bn, Hkv, G, d, C, seed):
    """Seeded cache contents, decode queries and fill counts (bf16 bits), on the GPU and on the host."""
    import torch

    from future_attention_targets_b200.workloads import f32_to_bf16_bits
    rng = np.random.default_rng(seed)
    bits = {"k": f32_to_bf16_bits(rng.standard_normal((Bn, Hkv, C, d)).astype(np.float32)),
            "v": f32_to_bf16_bits(rng.standard_normal((Bn, Hkv, C, d)).astype(np.float32)),
            "q": f32_to_bf16_bits(rng.standard_normal((Bn, Hkv * G, d)).astype(np.float32))}
    count = rng.integers(0, C + 1, size=(Bn, Hkv)).astype(np.int32)
    count[0, 0] = C          # one full cache row and one empty one
    count[-1, -1] = 0
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    dev = {k: to_dev(v) for k, v in bits.items()}
    dev["count"] = torch.from_numpy(count).cuda()
    return bits, count, dev


def _check_against(out, lse, ref_out, ref_lse, what):
    finite = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), finite), what
    assert float(np.max(np.abs(lse[finite] - ref_lse[finite]), initial=0.0)) <= LSE_TOL, what
    assert _rel_err(out, ref_out) <= TOL, what


def run_checks():
    import torch

    import oracle
    from future_attention_targets_b200 import _binding as B
    lib = B.lib()
    stream = torch.cuda.current_stream().cuda_stream
    shapes = [(7, 8, 4, 128, 4032, 2024),    # 3.7 MB of partials: most of the fixed 4 MiB array
              (1, 4, 4, 128, 1000, 7)]       # then a smaller shape over the larger one's leftovers
    cases = []
    for Bn, Hkv, G, d, C, seed in shapes:
        bits, count, dv = _case(Bn, Hkv, G, d, C, seed)
        shape = B.CacheShape(Bn, Hkv * G, Hkv, d, C)
        assert lib.kvpop_decode_workspace_bytes(shape) <= SCRATCH
        scale = 1.0 / math.sqrt(d)
        ref_out, ref_lse = oracle.decode_attention(bits["q"], bits["k"], bits["v"], count, scale)
        ws = torch.empty(lib.kvpop_decode_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
        w_out = torch.empty((Bn, Hkv * G, d), dtype=torch.float32, device="cuda")
        w_lse = torch.empty((Bn, Hkv * G), dtype=torch.float32, device="cuda")
        outs = [(torch.empty_like(w_out), torch.empty_like(w_lse)) for _ in range(2)]
        cases.append((shape, scale, dv, ref_out, ref_lse, ws, w_out, w_lse, outs))

    def noalloc(shape, scale, dv, out, lse):
        st = lib.kvpop_decode_attention_noalloc(dv["q"].data_ptr(), dv["k"].data_ptr(), dv["v"].data_ptr(),
                                                dv["count"].data_ptr(), shape, scale, out.data_ptr(),
                                                lse.data_ptr(), stream)
        assert st == B.OK, lib.kvpop_last_error()

    def workspace_version(shape, scale, dv, ws, out, lse):
        st = lib.kvpop_decode_attention(dv["q"].data_ptr(), dv["k"].data_ptr(), dv["v"].data_ptr(),
                                        dv["count"].data_ptr(), shape, scale, out.data_ptr(), lse.data_ptr(),
                                        ws.data_ptr(), ws.numel(), stream)
        assert st == B.OK, lib.kvpop_last_error()

    # Warm-up, before any free-memory reading: the first call on the device looks up the array's address,
    # and the first launch of each torch kernel used below (fill, copy to host) loads it lazily, which
    # takes device memory of its own.
    shape, scale, dv, _, _, ws, w_out, w_lse, outs = cases[0]
    noalloc(shape, scale, dv, *outs[0])
    workspace_version(shape, scale, dv, ws, w_out, w_lse)
    outs[0][0].fill_(float("nan"))
    outs[0][1].fill_(float("nan"))
    outs[0][0].cpu()
    torch.cuda.synchronize()
    for shape, scale, dv, ref_out, ref_lse, ws, w_out, w_lse, outs in cases:
        for out, lse in outs:
            out.fill_(float("nan"))
            lse.fill_(float("nan"))
        torch.cuda.synchronize()
        free_before, _ = torch.cuda.mem_get_info()
        for out, lse in outs:                # two calls in a row, nothing else in between
            noalloc(shape, scale, dv, out, lse)
        torch.cuda.synchronize()
        free_after, _ = torch.cuda.mem_get_info()
        assert free_after >= free_before, (shape.batch, free_before, free_after)
        workspace_version(shape, scale, dv, ws, w_out, w_lse)
        torch.cuda.synchronize()
        for call, (out, lse) in enumerate(outs):
            what = f"batch {shape.batch}, capacity {shape.capacity}, call {call}"
            o, l = out.cpu().numpy(), lse.cpu().numpy()
            _check_against(o, l, w_out.cpu().numpy(), w_lse.cpu().numpy(), what + " vs workspace version")
            _check_against(o, l, ref_out, ref_lse, what + " vs oracle")


@pytest.mark.gpu
def test_noalloc_decode_twice_against_workspace_version_and_oracle():
    run_checks()


@pytest.mark.gpu
def test_noalloc_decode_in_a_fresh_process():
    r = subprocess.run([sys.executable, os.path.abspath(__file__)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "NOALLOC_OK" in r.stdout, (r.stdout[-2000:], r.stderr[-4000:])


if __name__ == "__main__":
    run_checks()
    print("NOALLOC_OK")

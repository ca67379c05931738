"""The entry points inside CUDA graphs: stream capture once, then replay.

Every call is stream-ordered and, given its buffers and workspaces, allocates
nothing and never synchronises, so a whole step can be captured and replayed
as one graph launch.  A replay must reproduce the eager call bit for bit,
and a replay after new inputs were copied into the captured buffers must
equal an eager call on those inputs.
"""
import numpy as np
import pytest
import torch

from future_attention_targets_b200 import (check_status, decode_attention, decode_workspace_bytes, fused_workspace,
                                           future_targets, future_targets_fused, target_workspace_bytes)
from future_attention_targets_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _capture(fn):
    """Runs fn once on a side stream (first-launch setup), then captures it."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    return graph


def _replays_match(graph, eager, outs, refill, status=None):
    """Replays twice: on the captured inputs, then after refill() put new inputs in the captured buffers."""
    for step in range(2):
        if step == 1:
            refill()
        ref = [x.clone() for x in eager()]
        torch.cuda.synchronize()
        for x in outs:
            x.fill_(7)
        graph.replay()
        torch.cuda.synchronize()
        if status is not None:
            check_status(status)
        for a, b in zip(outs, ref):
            assert torch.equal(a, b)


@pytest.mark.parametrize("fused", [False, True], ids=["two_launch", "single_launch"])
def test_attention_pipeline_in_a_graph(fused):
    d = make_inputs("qwen3_4b_4k")
    w = d["workload"]
    q, k = dev(d["q_bits"]), dev(d["k_bits"])
    T = q.shape[0]
    cu, W, S, budgets, scale = d["cu_seqlens"], d["window"], d["sinks"], d["budgets"], d["scale"]
    lse = torch.empty((w.n_q_heads, T), dtype=torch.float32, device="cuda")
    tgt = torch.empty((w.n_kv_heads, T), dtype=torch.float32, device="cuda")
    keep = torch.empty((w.n_kv_heads, T), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if fused:
        ws = fused_workspace(cu, w.n_q_heads, w.n_kv_heads, w.head_dim)
        run = lambda: future_targets_fused(q, k, cu, W, S, budgets, scale=scale, lse=lse, target=tgt, keep=keep,
                                           workspace=ws, status=status)
    else:
        ws = torch.empty(target_workspace_bytes(T, w.n_q_heads, w.n_kv_heads, w.head_dim), dtype=torch.uint8,
                         device="cuda")
        run = lambda: future_targets(q, k, cu, W, S, budgets, scale=scale, lse=lse, target=tgt, keep=keep,
                                     workspace=ws, status=status)
    graph = _capture(run)
    other = make_inputs("qwen3_4b_4k", seed=5)

    def refill():
        q.copy_(dev(other["q_bits"]))
        k.copy_(dev(other["k_bits"]))

    # The eager reference runs the same entry point on separate outputs (and, for the single launch, its own
    # workspace).
    ws_eager = fused_workspace(cu, w.n_q_heads, w.n_kv_heads, w.head_dim) if fused else None

    def eager():
        if fused:
            return future_targets_fused(q, k, cu, W, S, budgets, scale=scale, workspace=ws_eager)
        return future_targets(q, k, cu, W, S, budgets, scale=scale)

    _replays_match(graph, eager, (lse, tgt, keep), refill, status)


def test_decode_step_in_a_graph():
    torch.manual_seed(0)
    B, Hq, Hkv, d, C = 4, 32, 8, 128, 1000
    q = torch.randn(B, Hq, d, device="cuda").to(torch.bfloat16)
    kc = torch.randn(B, Hkv, C, d, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B, Hkv, C, d, device="cuda").to(torch.bfloat16)
    cnt = torch.randint(1, C + 1, (B, Hkv), dtype=torch.int32, device="cuda")
    out = torch.empty(B, Hq, d, device="cuda")
    lse = torch.empty(B, Hq, device="cuda")
    ws = torch.empty(decode_workspace_bytes(B, Hq, Hkv, d, C), dtype=torch.uint8, device="cuda")
    graph = _capture(lambda: decode_attention(q, kc, vc, cnt, out=out, lse=lse, workspace=ws))

    def refill():
        q.copy_(torch.randn_like(q, dtype=torch.float32).to(torch.bfloat16))
        cnt.copy_(torch.randint(1, C + 1, (B, Hkv), dtype=torch.int32, device="cuda"))

    _replays_match(graph, lambda: decode_attention(q, kc, vc, cnt), (out, lse), refill)


def test_targets_compaction_decode_chain_in_a_graph():
    """Keep mask -> compaction -> decode in one graph.  The compaction and decode kernels are launched as
    programmatic dependents of the kernel before them; a replay after new Q/K/V and decode queries were
    copied in must still see the new keep mask and cache (their waits order them after their producers)."""
    from future_attention_targets_b200 import compact_kv
    from future_attention_targets_b200.workloads import random_qk
    d = make_inputs("qwen3_4b_4k")
    w = d["workload"]
    q, k = dev(d["q_bits"]), dev(d["k_bits"])
    T = q.shape[0]
    cu, W, S, budgets, scale = d["cu_seqlens"], d["window"], d["sinks"], d["budgets"], d["scale"]
    C = int(max(budgets))
    nb = len(cu) - 1
    v_bits, _ = random_qk(T, w.n_kv_heads, w.n_kv_heads, w.head_dim, seed=3)
    v = dev(v_bits)
    qd_bits, _ = random_qk(nb, w.n_q_heads, w.n_kv_heads, w.head_dim, seed=4)
    qd = dev(qd_bits.reshape(nb, w.n_q_heads, w.head_dim))
    lse = torch.empty((w.n_q_heads, T), dtype=torch.float32, device="cuda")
    tgt = torch.empty((w.n_kv_heads, T), dtype=torch.float32, device="cuda")
    keep = torch.empty((w.n_kv_heads, T), dtype=torch.uint8, device="cuda")
    cache = (torch.empty((nb, w.n_kv_heads, C, w.head_dim), dtype=torch.bfloat16, device="cuda"),
             torch.empty((nb, w.n_kv_heads, C, w.head_dim), dtype=torch.bfloat16, device="cuda"),
             torch.empty((nb, w.n_kv_heads, C), dtype=torch.int32, device="cuda"),
             torch.empty((nb, w.n_kv_heads), dtype=torch.int32, device="cuda"))
    out = torch.empty((nb, w.n_q_heads, w.head_dim), device="cuda")
    dl = torch.empty((nb, w.n_q_heads), device="cuda")
    ws = torch.empty(target_workspace_bytes(T, w.n_q_heads, w.n_kv_heads, w.head_dim), dtype=torch.uint8,
                     device="cuda")
    wsd = torch.empty(decode_workspace_bytes(nb, w.n_q_heads, w.n_kv_heads, w.head_dim, C), dtype=torch.uint8,
                      device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run():
        future_targets(q, k, cu, W, S, budgets, scale=scale, lse=lse, target=tgt, keep=keep, workspace=ws,
                       status=status)
        compact_kv(k, v, keep, cu, C, out=cache)
        decode_attention(qd, cache[0], cache[1], cache[3], scale, out=out, lse=dl, workspace=wsd)

    graph = _capture(run)
    other = make_inputs("qwen3_4b_4k", seed=9)
    v2_bits, _ = random_qk(T, w.n_kv_heads, w.n_kv_heads, w.head_dim, seed=10)
    qd2_bits, _ = random_qk(nb, w.n_q_heads, w.n_kv_heads, w.head_dim, seed=11)

    def refill():
        q.copy_(dev(other["q_bits"]))
        k.copy_(dev(other["k_bits"]))
        v.copy_(dev(v2_bits))
        qd.copy_(dev(qd2_bits.reshape(nb, w.n_q_heads, w.head_dim)))

    def eager():
        _, _, kp = future_targets(q, k, cu, W, S, budgets, scale=scale)
        kc, vc, pos, cnt = compact_kv(k, v, kp, cu, C)
        o, l = decode_attention(qd, kc, vc, cnt, scale)
        return kp, kc, vc, pos, cnt, o, l

    _replays_match(graph, eager, (keep,) + cache + (out, dl), refill, status)

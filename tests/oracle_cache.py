"""Full-size oracle results for the large workloads, computed once and kept on disk.

TEST INFRASTRUCTURE: this module calls only the CPU oracle (``oracle/``) and
the seeded input generators (``workloads.py``, which hold none of the
method's arithmetic).  Nothing here comes from the CUDA path.

For every KV head h of a workload it runs ``oracle.future_target`` on K head
h and its G query heads over all positions (the oracle's own materialised
fp64 softmax), and keeps
  target   [H_kv, T]  float64  every key's future-attention target
  lse      [H_q, T]   float64  every row's natural-log logsumexp
  far_sum  [H_kv, B]  float64  per sequence, the sum over the group's query
                               heads and rows of the mass each query puts on
                               keys at least W back (the mass-conservation
                               invariant: it must equal the sum of the
                               targets of that sequence and KV head).

KV heads are independent problems, so they run in parallel worker processes
(started with ``spawn``, one BLAS thread each).  Results are cached under
``tests/.oracle_cache/`` (git-ignored), keyed by the workload name, its seed,
a hash of the exact input bits, window and scale, and a hash of the oracle's
source, so a change to either recomputes them.

    python tests/oracle_cache.py qwen3_8b_16k varlen_8x long_64k
"""
from __future__ import annotations

import hashlib
import multiprocessing as mp
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

CACHE_DIR = os.path.join(ROOT, "tests", ".oracle_cache")
ORACLE_SRC = os.path.join(ROOT, "oracle", "kvpop_oracle.py")


def _key(d: dict) -> str:
    h = hashlib.sha256()
    for name in ("q_bits", "k_bits", "cu_seqlens"):
        h.update(np.ascontiguousarray(d[name]).tobytes())
    h.update(repr((int(d["window"]), float(d["scale"]))).encode())
    with open(ORACLE_SRC, "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:20]


def _one_head(args):
    """Worker: the oracle on one KV head (its K column and G query heads)."""
    q_grp, k_head, cu, window, scale = args
    from threadpoolctl import threadpool_limits

    import oracle
    with threadpool_limits(1):
        tgt, lse, far = oracle.future_target(q_grp, k_head, cu, window, scale, return_lse=True, return_far=True)
    cu = np.asarray(cu, dtype=np.int64)
    far_sum = np.array([float(np.sum(far[:, cu[b]:cu[b + 1]])) for b in range(len(cu) - 1)])
    return tgt[0], lse, far_sum


def compute(d: dict, workers: int | None = None) -> dict:
    """Oracle target, lse and far-mass sums for every KV head of the inputs ``d`` (no cache)."""
    w = d["workload"]
    G, Hkv = w.group, w.n_kv_heads
    tasks = [(np.ascontiguousarray(d["q_bits"][:, h * G:(h + 1) * G]),
              np.ascontiguousarray(d["k_bits"][:, h:h + 1]),
              d["cu_seqlens"], d["window"], d["scale"]) for h in range(Hkv)]
    n = max(1, min(Hkv, workers or os.cpu_count() or 1))
    if n == 1:
        parts = [_one_head(t) for t in tasks]
    else:
        with mp.get_context("spawn").Pool(n) as pool:
            parts = pool.map(_one_head, tasks, chunksize=1)
    return {"target": np.stack([p[0] for p in parts]),
            "lse": np.concatenate([p[1] for p in parts]),
            "far_sum": np.stack([p[2] for p in parts])}


def oracle_full(name: str, d: dict | None = None, seed: int | None = None) -> dict:
    """Cached full-size oracle results of workload ``name`` (inputs drawn here unless given)."""
    from future_attention_targets_b200.workloads import make_inputs
    if d is None:
        d = make_inputs(name, seed=seed)
    key = _key(d)
    path = os.path.join(CACHE_DIR, f"{name}-seed{d['workload'].seed}-{key}.npz")
    if os.path.exists(path):
        with np.load(path) as z:
            return {k: z[k] for k in ("target", "lse", "far_sum")}
    res = compute(d)
    os.makedirs(CACHE_DIR, exist_ok=True)
    tmp = path + f".{os.getpid()}.tmp.npz"
    np.savez(tmp, **res)
    os.replace(tmp, path)
    return res


if __name__ == "__main__":
    for nm in sys.argv[1:] or ["qwen3_8b_16k", "varlen_8x", "long_64k"]:
        t0 = time.perf_counter()
        r = oracle_full(nm)
        print(f"{nm}: target {r['target'].shape}, lse {r['lse'].shape} in {time.perf_counter() - t0:.1f} s",
              flush=True)

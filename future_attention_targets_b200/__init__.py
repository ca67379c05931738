"""KVpop future-attention targets on NVIDIA B200 (sm_100a).

The compute lives in libkvpop.so (C ABI in include/kvpop.h, CUDA kernels in
csrc/); this package is its Python binding plus the seeded workload
generators.  See ``_binding`` for the entry points.
"""
from ._binding import (  # noqa: F401
    HostPipeline,
    KvpopError,
    check_status,
    compact_kv,
    debug_selftest,
    debug_set_word,
    decode_attention,
    decode_workspace_bytes,
    future_target,
    future_target_split,
    future_targets,
    future_targets_fused,
    fused_workspace,
    keep_mask,
    lib,
    prefix_topk_thresholds,
    row_lse,
    selftest_bounded_wait,
    target_split_workspace_bytes,
    target_workspace_bytes,
)

__all__ = ["HostPipeline", "KvpopError", "check_status", "compact_kv", "debug_selftest", "debug_set_word",
           "decode_attention",
           "decode_workspace_bytes", "future_target", "future_target_split", "future_targets", "future_targets_fused",
           "fused_workspace", "keep_mask", "lib", "prefix_topk_thresholds", "row_lse", "selftest_bounded_wait",
           "target_split_workspace_bytes", "target_workspace_bytes"]

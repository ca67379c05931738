"""CPU float64 oracle for KVpop future-attention targets (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
may import this package; the CUDA library never does.
"""
from .kvpop_oracle import (ROW_BLOCK, as_f64, compact_kv, decode_attention, future_target, keep_mask,
                           prefix_topk_thresholds, row_lse)

__all__ = ["ROW_BLOCK", "as_f64", "compact_kv", "decode_attention", "future_target", "keep_mask",
           "prefix_topk_thresholds", "row_lse"]

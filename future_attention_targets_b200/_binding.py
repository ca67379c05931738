"""ctypes binding of libkvpop.so (include/kvpop.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; PyTorch is
used here only to allocate device memory and to supply the current stream.
There is no CPU fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import re
import threading

import numpy as np

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libkvpop.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG_DIR), "include", "kvpop.h")

DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libkvpop_debug.so")

OK, INVALID_ARG, UNSUPPORTED, CUDA_ERROR, TIMEOUT, BOUNDS = 0, 1, 2, 3, 4, 5
STATUS_NAMES = {OK: "KVPOP_OK", INVALID_ARG: "KVPOP_ERR_INVALID_ARG", UNSUPPORTED: "KVPOP_ERR_UNSUPPORTED",
                CUDA_ERROR: "KVPOP_ERR_CUDA", TIMEOUT: "KVPOP_ERR_TIMEOUT", BOUNDS: "KVPOP_ERR_BOUNDS"}


class KvpopError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("total_tokens", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class CacheShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("capacity", ctypes.c_int32)]


_P = ctypes.c_void_p
_I32P = ctypes.POINTER(ctypes.c_int32)
_SIGS = {
    "kvpop_row_lse": (ctypes.c_int, [_P, _P, _I32P, Shape, ctypes.c_float, _P, _P, _P]),
    "kvpop_target_workspace_bytes": (ctypes.c_size_t, [Shape]),
    "kvpop_future_target": (ctypes.c_int, [_P, _P, _I32P, Shape, ctypes.c_float, ctypes.c_int32, _P, _P, _P,
                                           ctypes.c_size_t, _P, _P]),
    "kvpop_keep_mask": (ctypes.c_int, [_P, _I32P, Shape, ctypes.c_int32, ctypes.c_int32, _I32P, _P, _P]),
    "kvpop_prefix_topk_thresholds": (ctypes.c_int, [_P, _I32P, Shape, ctypes.c_int32, ctypes.c_int32, _I32P, _P,
                                                    _P, _P]),
    "kvpop_compact_kv": (ctypes.c_int, [_P, _P, _P, _I32P, Shape, ctypes.c_int32, _P, _P, _P, _P, _P]),
    "kvpop_decode_workspace_bytes": (ctypes.c_size_t, [CacheShape]),
    "kvpop_decode_attention": (ctypes.c_int, [_P, _P, _P, _P, CacheShape, ctypes.c_float, _P, _P, _P, ctypes.c_size_t,
                                              _P]),
    "kvpop_decode_attention_noalloc": (ctypes.c_int, [_P, _P, _P, _P, CacheShape, ctypes.c_float, _P, _P, _P]),
    "kvpop_future_targets": (ctypes.c_int, [_P, _P, _I32P, Shape, ctypes.c_float, ctypes.c_int32, ctypes.c_int32,
                                            _I32P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "kvpop_target_split_workspace_bytes": (ctypes.c_size_t, [Shape]),
    "kvpop_future_target_split": (ctypes.c_int, [_P, _P, _I32P, Shape, ctypes.c_float, ctypes.c_int32, _P, _P, _P,
                                                 ctypes.c_size_t, _P, _P]),
    "kvpop_fused_workspace_bytes": (ctypes.c_size_t, [_I32P, Shape]),
    "kvpop_future_targets_fused": (ctypes.c_int, [_P, _P, _I32P, Shape, ctypes.c_float, ctypes.c_int32,
                                                  ctypes.c_int32, _I32P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "kvpop_host_workspace_bytes": (ctypes.c_size_t, [Shape]),
    "kvpop_future_targets_host": (ctypes.c_int, [_P, _P, _I32P, Shape, ctypes.c_float, ctypes.c_int32,
                                                 ctypes.c_int32, _I32P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "kvpop_check_device_status": (ctypes.c_int, [_P, _P]),
    "kvpop_selftest_bounded_wait": (ctypes.c_int, [_P, ctypes.c_uint64, _P]),
    "kvpop_debug_set_word": (ctypes.c_int, [_P]),
    "kvpop_debug_selftest": (ctypes.c_int, [_P, _P]),
    "kvpop_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kvpop_last_error": (ctypes.c_char_p, []),
    "kvpop_abi_version": (ctypes.c_int32, []),
}

_lock = threading.Lock()
_handle = None


def lib() -> ctypes.CDLL:
    """Loads libkvpop.so (once).  Raises if it has not been built."""
    global _handle
    with _lock:
        if _handle is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m future_attention_targets_b200.build` (needs nvcc)")
            h = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                fn = getattr(h, name)
                fn.restype = res
                fn.argtypes = args
            _handle = h
    return _handle


def use_library(path: str) -> str:
    """Makes later calls go to another build of the same C ABI (for example the
    bounds-checking debug build, DEBUG_LIB_PATH); returns the previous path.
    The library at `path` must exist: nothing falls back to anything else."""
    global LIB_PATH, _handle
    with _lock:
        old = LIB_PATH
        LIB_PATH, _handle = path, None
    lib()
    return old


def header_symbols() -> list[str]:
    """Entry points declared in include/kvpop.h."""
    with open(HEADER_PATH) as f:
        return re.findall(r"KVPOP_API\s+[\w\s\*]+?\b(kvpop_\w+)\s*\(", f.read())


def _check(status: int) -> None:
    if status != OK:
        raise KvpopError(status, lib().kvpop_last_error().decode())


def _i32_host(values) -> ctypes.Array:
    arr = np.ascontiguousarray(np.asarray(values, dtype=np.int64))
    if arr.size and (arr.min() < -2**31 or arr.max() >= 2**31):
        raise ValueError("value out of int32 range")
    return (ctypes.c_int32 * arr.size)(*arr.astype(np.int32).tolist())


def _cu_host(cu_seqlens):
    try:
        import torch
        if isinstance(cu_seqlens, torch.Tensor):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    cu = np.asarray(cu_seqlens, dtype=np.int64).reshape(-1)
    return cu, _i32_host(cu)


def _stream_ptr(stream) -> int:
    """The raw cudaStream_t of `stream` (a torch.cuda.Stream, a raw handle, or None for the current stream).
    A torch stream must belong to the current device, on which the library launches."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    if hasattr(stream, "cuda_stream"):
        dev = getattr(stream, "device", None)
        cur = torch.cuda.current_device()
        if dev is not None and dev.index is not None and dev.index != cur:
            raise ValueError(f"stream belongs to {dev} but the current CUDA device is cuda:{cur}")
        return int(stream.cuda_stream)
    return int(stream)


def _on_current_device(t, name) -> None:
    """The library launches on the calling thread's current CUDA device and takes raw pointers, so every
    tensor it is given must live on that device (a pointer into another GPU would be read as a peer
    address)."""
    import torch
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device} but the current CUDA device is cuda:{cur}; "
                         f"call under torch.cuda.device({t.device})")


def _status_ptr(status, device):
    """Pointer of the optional int32 status word (a CUDA tensor on `device` with at least one element)."""
    import torch
    if status is None:
        return None
    if (not isinstance(status, torch.Tensor) or status.dtype != torch.int32 or not status.is_cuda
            or status.device != device or status.numel() < 1):
        raise ValueError(f"status must be an int32 CUDA tensor on {device} with at least one element")
    return status.data_ptr()


def _shape(q, k, cu) -> Shape:
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    return Shape(len(cu) - 1, T, Hq, Hkv, d)


def _check_qk(q, k):
    import torch
    for name, t in (("q", q), ("k", k)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 3:
            raise TypeError(f"{name} must be a 3-D bf16 CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.shape[0] != k.shape[0] or q.shape[2] != k.shape[2]:
        raise ValueError("q [T, H_q, d] and k [T, H_kv, d] disagree on T or d")
    if k.device != q.device:
        raise ValueError(f"q is on {q.device} and k on {k.device}")
    _on_current_device(q, "q")


def _tensor(t, shape, dtype, device, name):
    """t, checked: the kernels read or write it through its pointer alone, so its dtype, shape, device and
    layout must be exactly what the call describes."""
    import torch
    if (not isinstance(t, torch.Tensor) or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_cuda
            or t.device != device or not t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous {dtype} CUDA tensor of shape {tuple(shape)} on {device}")
    return t


def _out(t, shape, dtype, device, name):
    """A fresh output tensor when t is None, else t after _tensor's checks."""
    import torch
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return _tensor(t, shape, dtype, device, name)


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


# ------------------------------------------------------------------ entry points

def row_lse(q, k, cu_seqlens, scale: float | None = None, out=None, status=None, stream=None):
    """lse [H_q, T] fp32 (natural log) of the causal softmax rows."""
    import torch
    _check_qk(q, k)
    cu, cu_c = _cu_host(cu_seqlens)
    sh = _shape(q, k, cu)
    scale = 1.0 / math.sqrt(sh.head_dim) if scale is None else float(scale)
    out = _out(out, (sh.n_q_heads, sh.total_tokens), torch.float32, q.device, "out")
    _check(lib().kvpop_row_lse(q.data_ptr(), k.data_ptr(), cu_c, sh, scale, out.data_ptr(),
                               _status_ptr(status, q.device), _stream_ptr(stream)))
    return out


def _workspace(nbytes: int, device, workspace):
    """The caller's workspace (a contiguous CUDA tensor on `device`; the library checks its size in bytes)
    if given, else a fresh uint8 CUDA tensor of nbytes (at least 256)."""
    import torch
    if workspace is None:
        return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    if (not isinstance(workspace, torch.Tensor) or not workspace.is_cuda or workspace.device != device
            or not workspace.is_contiguous()):
        raise ValueError(f"workspace must be a contiguous CUDA tensor on {device}")
    return workspace


def future_target(q, k, cu_seqlens, window: int, lse, scale: float | None = None, out=None, workspace=None,
                  status=None, stream=None):
    """target [H_kv, T] fp32: mass each key receives from queries i >= j + W, summed over its GQA group."""
    import torch
    _check_qk(q, k)
    cu, cu_c = _cu_host(cu_seqlens)
    sh = _shape(q, k, cu)
    scale = 1.0 / math.sqrt(sh.head_dim) if scale is None else float(scale)
    _tensor(lse, (sh.n_q_heads, sh.total_tokens), torch.float32, q.device, "lse")
    out = _out(out, (sh.n_kv_heads, sh.total_tokens), torch.float32, q.device, "out")
    workspace = _workspace(lib().kvpop_target_workspace_bytes(sh), q.device, workspace)
    _check(lib().kvpop_future_target(q.data_ptr(), k.data_ptr(), cu_c, sh, scale, int(window),
                                     lse.data_ptr(), out.data_ptr(), workspace.data_ptr(),
                                     _nbytes(workspace), _status_ptr(status, q.device), _stream_ptr(stream)))
    return out


def future_target_split(q, k, cu_seqlens, window: int, lse, scale: float | None = None, out=None, workspace=None,
                        status=None, stream=None):
    """future_target with one item per (key tile, query head); bit-identical result, for few KV heads per call."""
    import torch
    _check_qk(q, k)
    cu, cu_c = _cu_host(cu_seqlens)
    sh = _shape(q, k, cu)
    scale = 1.0 / math.sqrt(sh.head_dim) if scale is None else float(scale)
    _tensor(lse, (sh.n_q_heads, sh.total_tokens), torch.float32, q.device, "lse")
    out = _out(out, (sh.n_kv_heads, sh.total_tokens), torch.float32, q.device, "out")
    workspace = _workspace(lib().kvpop_target_split_workspace_bytes(sh), q.device, workspace)
    _check(lib().kvpop_future_target_split(q.data_ptr(), k.data_ptr(), cu_c, sh, scale, int(window),
                                           lse.data_ptr(), out.data_ptr(), workspace.data_ptr(),
                                           _nbytes(workspace), _status_ptr(status, q.device), _stream_ptr(stream)))
    return out


def target_workspace_bytes(total_tokens: int, n_q_heads: int, n_kv_heads: int, head_dim: int) -> int:
    """Device workspace of future_target and future_targets (the transposed pass's normaliser rows)."""
    return int(lib().kvpop_target_workspace_bytes(Shape(1, total_tokens, n_q_heads, n_kv_heads, head_dim)))


def target_split_workspace_bytes(total_tokens: int, n_q_heads: int, n_kv_heads: int, head_dim: int) -> int:
    return int(lib().kvpop_target_split_workspace_bytes(Shape(1, total_tokens, n_q_heads, n_kv_heads, head_dim)))


def keep_mask(score, cu_seqlens, window: int, sinks: int, budgets, out=None, stream=None):
    """keep [H_kv, T] uint8: sinks + recent window + top-(budget - sinks - window) scores."""
    import torch
    if score.dtype != torch.float32 or not score.is_cuda or score.dim() != 2 or not score.is_contiguous():
        raise TypeError("score must be a contiguous 2-D fp32 CUDA tensor [H_kv, T]")
    _on_current_device(score, "score")
    cu, cu_c = _cu_host(cu_seqlens)
    Hkv, T = score.shape
    sh = Shape(len(cu) - 1, T, Hkv, Hkv, 128)
    bud = _i32_host(budgets)
    if len(bud) != sh.batch:
        raise ValueError("one budget per sequence is needed")
    out = _out(out, (Hkv, T), torch.uint8, score.device, "out")
    _check(lib().kvpop_keep_mask(score.data_ptr(), cu_c, sh, int(window), int(sinks), bud, out.data_ptr(),
                                 _stream_ptr(stream)))
    return out


def prefix_topk_thresholds(score, cu_seqlens, window: int, sinks: int, budgets, out=None, stream=None):
    """Per-step eviction thresholds: (thr_score fp32 [H_kv, T], thr_pos int32 [H_kv, T])."""
    import torch
    if score.dtype != torch.float32 or not score.is_cuda or score.dim() != 2 or not score.is_contiguous():
        raise TypeError("score must be a contiguous 2-D fp32 CUDA tensor [H_kv, T]")
    _on_current_device(score, "score")
    cu, cu_c = _cu_host(cu_seqlens)
    Hkv, T = score.shape
    sh = Shape(len(cu) - 1, T, Hkv, Hkv, 128)
    bud = _i32_host(budgets)
    if len(bud) != sh.batch:
        raise ValueError("one budget per sequence is needed")
    out = (None, None) if out is None else out
    thr_s = _out(out[0], (Hkv, T), torch.float32, score.device, "out[0]")
    thr_p = _out(out[1], (Hkv, T), torch.int32, score.device, "out[1]")
    _check(lib().kvpop_prefix_topk_thresholds(score.data_ptr(), cu_c, sh, int(window), int(sinks), bud,
                                              thr_s.data_ptr(), thr_p.data_ptr(), _stream_ptr(stream)))
    return thr_s, thr_p


def compact_kv(k, v, keep, cu_seqlens, capacity: int, out=None, stream=None):
    """Static cache: (k_cache, v_cache [B, H_kv, C, d] bf16, pos [B, H_kv, C] int32, count [B, H_kv] int32)."""
    import torch
    for name, t in (("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 3 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous 3-D bf16 CUDA tensor [T, H_kv, d]")
    _on_current_device(k, "k")
    cu, cu_c = _cu_host(cu_seqlens)
    T, Hkv, d = k.shape
    _tensor(v, (T, Hkv, d), torch.bfloat16, k.device, "v")
    _tensor(keep, (Hkv, T), torch.uint8, k.device, "keep")
    B = len(cu) - 1
    sh = Shape(B, T, Hkv, Hkv, d)
    out = (None,) * 4 if out is None else out
    kc = _out(out[0], (B, Hkv, capacity, d), torch.bfloat16, k.device, "out[0]")
    vc = _out(out[1], (B, Hkv, capacity, d), torch.bfloat16, k.device, "out[1]")
    pos = _out(out[2], (B, Hkv, capacity), torch.int32, k.device, "out[2]")
    cnt = _out(out[3], (B, Hkv), torch.int32, k.device, "out[3]")
    _check(lib().kvpop_compact_kv(k.data_ptr(), v.data_ptr(), keep.data_ptr(), cu_c, sh, int(capacity),
                                  kc.data_ptr(), vc.data_ptr(), pos.data_ptr(), cnt.data_ptr(), _stream_ptr(stream)))
    return kc, vc, pos, cnt


def decode_workspace_bytes(batch, n_q_heads, n_kv_heads, head_dim, capacity) -> int:
    return int(lib().kvpop_decode_workspace_bytes(CacheShape(batch, n_q_heads, n_kv_heads, head_dim, capacity)))


def decode_attention(q, k_cache, v_cache, count, scale: float | None = None, out=None, lse=None, workspace=None,
                     stream=None):
    """One decode step over the compacted cache: (out [B, H_q, d] fp32, lse [B, H_q] fp32)."""
    import torch
    if q.dtype != torch.bfloat16 or not q.is_cuda or q.dim() != 3 or not q.is_contiguous():
        raise TypeError("q must be a contiguous 3-D bf16 CUDA tensor [B, H_q, d]")
    _on_current_device(q, "q")
    B, Hq, d = q.shape
    if not isinstance(k_cache, torch.Tensor) or k_cache.dim() != 4:
        raise TypeError("k_cache must be a 4-D bf16 CUDA tensor [B, H_kv, C, d]")
    _, Hkv, C, _ = k_cache.shape
    _tensor(k_cache, (B, Hkv, C, d), torch.bfloat16, q.device, "k_cache")
    _tensor(v_cache, (B, Hkv, C, d), torch.bfloat16, q.device, "v_cache")
    _tensor(count, (B, Hkv), torch.int32, q.device, "count")
    sh = CacheShape(B, Hq, Hkv, d, C)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = _out(out, (B, Hq, d), torch.float32, q.device, "out")
    lse = _out(lse, (B, Hq), torch.float32, q.device, "lse")
    workspace = _workspace(lib().kvpop_decode_workspace_bytes(sh), q.device, workspace)
    _check(lib().kvpop_decode_attention(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), count.data_ptr(), sh,
                                        scale, out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                        _nbytes(workspace), _stream_ptr(stream)))
    return out, lse


def future_targets(q, k, cu_seqlens, window: int, sinks: int, budgets, scale: float | None = None,
                   lse=None, target=None, keep=None, workspace=None, status=None, stream=None):
    """The whole hot path on device tensors: returns (lse, target, keep)."""
    import torch
    _check_qk(q, k)
    cu, cu_c = _cu_host(cu_seqlens)
    sh = _shape(q, k, cu)
    scale = 1.0 / math.sqrt(sh.head_dim) if scale is None else float(scale)
    dev = q.device
    lse = _out(lse, (sh.n_q_heads, sh.total_tokens), torch.float32, dev, "lse")
    target = _out(target, (sh.n_kv_heads, sh.total_tokens), torch.float32, dev, "target")
    keep = _out(keep, (sh.n_kv_heads, sh.total_tokens), torch.uint8, dev, "keep")
    bud = _i32_host(budgets)
    workspace = _workspace(lib().kvpop_target_workspace_bytes(sh), dev, workspace)
    _check(lib().kvpop_future_targets(q.data_ptr(), k.data_ptr(), cu_c, sh, scale, int(window), int(sinks), bud,
                                      lse.data_ptr(), target.data_ptr(), keep.data_ptr(), workspace.data_ptr(),
                                      _nbytes(workspace), _status_ptr(status, q.device), _stream_ptr(stream)))
    return lse, target, keep


def fused_workspace(cu_seqlens, n_q_heads: int, n_kv_heads: int, head_dim: int, device=None):
    """Zero-filled workspace for future_targets_fused: the flag counters (each completed call leaves them
    zeroed, so the workspace is reusable), then the normaliser rows (scratch)."""
    import torch
    cu, cu_c = _cu_host(cu_seqlens)
    sh = Shape(len(cu) - 1, int(cu[-1]), n_q_heads, n_kv_heads, head_dim)
    n = int(lib().kvpop_fused_workspace_bytes(cu_c, sh))
    if n == 0:
        raise ValueError("cu_seqlens / head counts do not describe a valid problem")
    return torch.zeros(n, dtype=torch.uint8, device=torch.device("cuda") if device is None else device)


def future_targets_fused(q, k, cu_seqlens, window: int, sinks: int, budgets, scale: float | None = None,
                         lse=None, target=None, keep=None, workspace=None, status=None, stream=None):
    """future_targets with both attention passes in one cooperative launch: returns (lse, target, keep)."""
    import torch
    _check_qk(q, k)
    cu, cu_c = _cu_host(cu_seqlens)
    sh = _shape(q, k, cu)
    scale = 1.0 / math.sqrt(sh.head_dim) if scale is None else float(scale)
    dev = q.device
    lse = _out(lse, (sh.n_q_heads, sh.total_tokens), torch.float32, dev, "lse")
    target = _out(target, (sh.n_kv_heads, sh.total_tokens), torch.float32, dev, "target")
    keep = _out(keep, (sh.n_kv_heads, sh.total_tokens), torch.uint8, dev, "keep")
    if workspace is None:
        workspace = fused_workspace(cu, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, device=dev)
    workspace = _workspace(0, dev, workspace)
    bud = _i32_host(budgets)
    _check(lib().kvpop_future_targets_fused(q.data_ptr(), k.data_ptr(), cu_c, sh, scale, int(window), int(sinks),
                                            bud, lse.data_ptr(), target.data_ptr(), keep.data_ptr(),
                                            workspace.data_ptr(), _nbytes(workspace),
                                            _status_ptr(status, q.device), _stream_ptr(stream)))
    return lse, target, keep


class HostPipeline:
    """The hot path on host buffers through kvpop_future_targets_host.

    Owns one device workspace (allocated once by torch) and pinned host
    outputs; each call copies q and k in, runs the three passes and copies
    target and keep out, all on one stream.
    """

    def __init__(self, cu_seqlens, n_q_heads: int, n_kv_heads: int, head_dim: int, window: int, sinks: int,
                 budgets, scale: float | None = None, device=None):
        import torch
        self.cu, self.cu_c = _cu_host(cu_seqlens)
        T = int(self.cu[-1])
        self.shape = Shape(len(self.cu) - 1, T, n_q_heads, n_kv_heads, head_dim)
        self.window, self.sinks = int(window), int(sinks)
        self.budgets = _i32_host(budgets)
        self.scale = 1.0 / math.sqrt(head_dim) if scale is None else float(scale)
        self.device = torch.device("cuda") if device is None else torch.device(device)
        nbytes = int(lib().kvpop_host_workspace_bytes(self.shape))
        self.workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.target = torch.empty((n_kv_heads, T), dtype=torch.float32, pin_memory=True)
        self.keep = torch.empty((n_kv_heads, T), dtype=torch.uint8, pin_memory=True)
        self.h2d_bytes = T * (n_q_heads + n_kv_heads) * head_dim * 2
        self.d2h_bytes = T * n_kv_heads * 5

    def submit(self, q_host, k_host, stream=None):
        """Enqueues one step on `stream` and returns at once; self.target and self.keep hold its results
        once the stream has reached this point.  The workspace is reused by the next call on the same
        stream only after this one's work there, so two pipelines on two streams let one step's copies in
        overlap the other's compute."""
        import torch
        T, Hq, Hkv, d = self.shape.total_tokens, self.shape.n_q_heads, self.shape.n_kv_heads, self.shape.head_dim
        for name, t, shape in (("q_host", q_host, (T, Hq, d)), ("k_host", k_host, (T, Hkv, d))):
            if (not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.is_cuda
                    or tuple(t.shape) != shape or not t.is_contiguous()):
                raise ValueError(f"{name} must be a contiguous bf16 CPU tensor of shape {shape}")
        _on_current_device(self.workspace, "the pipeline's workspace")
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        _check(lib().kvpop_future_targets_host(
            q_host.data_ptr(), k_host.data_ptr(), self.cu_c, self.shape, self.scale, self.window, self.sinks,
            self.budgets, self.target.data_ptr(), self.keep.data_ptr(), self.workspace.data_ptr(),
            self.workspace.numel(), self.status.data_ptr(), _stream_ptr(s)))
        return s

    def __call__(self, q_host, k_host, stream=None):
        """q_host, k_host: pinned CPU bf16 tensors.  Returns (target, keep) host tensors after syncing."""
        self.submit(q_host, k_host, stream).synchronize()
        return self.target, self.keep


def check_status(status, stream=None) -> None:
    """Raises KvpopError(TIMEOUT) when a kernel recorded a wait that ran out."""
    _on_current_device(status, "status")
    _check(lib().kvpop_check_device_status(_status_ptr(status, status.device), _stream_ptr(stream)))


def selftest_bounded_wait(status, limit_ns: int, stream=None) -> None:
    _on_current_device(status, "status")
    _check(lib().kvpop_selftest_bounded_wait(_status_ptr(status, status.device), int(limit_ns),
                                             _stream_ptr(stream)))


def debug_set_word(word) -> None:
    """Debug build: registers a zero-filled one-word int32 CUDA tensor that the kernels' bounds checks
    write (None stops recording).  The ordinary build raises KVPOP_ERR_UNSUPPORTED."""
    if word is None:
        _check(lib().kvpop_debug_set_word(None))
        return
    _on_current_device(word, "word")
    _check(lib().kvpop_debug_set_word(_status_ptr(word, word.device)))


def debug_selftest(word, stream=None) -> None:
    """Debug build: one kernel makes an index check that fails by design and records its code in word."""
    _on_current_device(word, "word")
    _check(lib().kvpop_debug_selftest(_status_ptr(word, word.device), _stream_ptr(stream)))

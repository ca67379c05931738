"""The C-ABI library on the CPU: it loads, exports every declared symbol, and
rejects bad arguments before any device call (no GPU needed)."""
import ctypes

import numpy as np
import pytest

from future_attention_targets_b200 import _binding as B
from future_attention_targets_b200.build import build


@pytest.fixture(scope="module")
def lib():
    build()
    return B.lib()


def test_exports_every_header_symbol(lib):
    names = B.header_symbols()
    assert len(names) == 23, names
    for name in names:
        assert hasattr(lib, name), f"{name} declared in kvpop.h but not exported"
    assert set(names) == set(B._SIGS), "binding signatures and header disagree"


def test_version_and_strings(lib):
    assert lib.kvpop_abi_version() == 3
    for code, word in [(0, b"ok"), (1, b"invalid argument"), (2, b"unsupported"), (3, b"CUDA error"),
                       (4, b"device wait timed out"), (5, b"a bounds check of the debug build failed")]:
        assert lib.kvpop_status_string(code) == word


def test_ordinary_build_has_no_bounds_checks(lib):
    """The debug calls exist in every build; the ordinary library refuses them before touching a device."""
    assert lib.kvpop_debug_set_word(FAKE) == B.UNSUPPORTED
    assert lib.kvpop_debug_selftest(FAKE, None) == B.UNSUPPORTED


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _shape(batch=1, T=100, hq=4, hkv=2, d=128):
    return B.Shape(batch, T, hq, hkv, d)


def _cu(*v):
    return B._i32_host(v)


def _row_lse(lib, q=FAKE, k=FAKE, cu=None, shape=None, scale=0.1, lse=FAKE):
    cu = _cu(0, 100) if cu is None else cu
    shape = _shape() if shape is None else shape
    return lib.kvpop_row_lse(q, k, cu, shape, scale, lse, None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), B.INVALID_ARG),
    (dict(k=None), B.INVALID_ARG),
    (dict(lse=None), B.INVALID_ARG),
    (dict(q=FAKE + 2), B.INVALID_ARG),                       # misaligned
    (dict(scale=float("nan")), B.INVALID_ARG),
    (dict(scale=float("inf")), B.INVALID_ARG),
    (dict(scale=0.0), B.INVALID_ARG),
    (dict(scale=-0.1), B.INVALID_ARG),
    (dict(shape=_shape(hq=3, hkv=2)), B.INVALID_ARG),         # H_q not a multiple of H_kv
    (dict(shape=_shape(hkv=0)), B.INVALID_ARG),
    (dict(shape=_shape(d=96)), B.UNSUPPORTED),
    (dict(shape=_shape(d=256)), B.UNSUPPORTED),
    (dict(shape=_shape(batch=0)), B.INVALID_ARG),
    (dict(shape=_shape(batch=513), cu=_cu(*([0] * 514))), B.UNSUPPORTED),
    (dict(shape=_shape(T=99)), B.INVALID_ARG),               # cu[batch] != T
    (dict(cu=_cu(1, 100)), B.INVALID_ARG),                    # cu[0] != 0
    (dict(shape=_shape(batch=2), cu=_cu(0, 60, 50)), B.INVALID_ARG),   # decreasing
    (dict(shape=_shape(T=131073), cu=_cu(0, 131073)), B.UNSUPPORTED),  # sequence too long
])
def test_row_lse_rejects(lib, kw, code):
    assert _row_lse(lib, **kw) == code
    assert lib.kvpop_last_error()


def test_cu_seqlens_null(lib):
    assert lib.kvpop_row_lse(FAKE, FAKE, None, _shape(), 0.1, FAKE, None, None) == B.INVALID_ARG


def test_future_target_rejects(lib):
    cu, sh = _cu(0, 100), _shape()
    need = lib.kvpop_target_workspace_bytes(sh)
    F = lib.kvpop_future_target
    assert F(FAKE, FAKE, cu, sh, 0.1, -1, FAKE, FAKE, FAKE, need, None, None) == B.INVALID_ARG      # window
    assert F(FAKE, FAKE, cu, sh, 0.1, 4, None, FAKE, FAKE, need, None, None) == B.INVALID_ARG       # lse
    assert F(FAKE, FAKE, cu, sh, 0.1, 4, FAKE, None, FAKE, need, None, None) == B.INVALID_ARG       # target
    assert F(FAKE, FAKE, cu, sh, 0.1, 4, FAKE, FAKE, None, need, None, None) == B.INVALID_ARG       # no workspace
    assert F(FAKE, FAKE, cu, sh, 0.1, 4, FAKE, FAKE, FAKE, need - 1, None, None) == B.INVALID_ARG   # too small
    assert F(FAKE, FAKE, cu, sh, 0.1, 4, FAKE, FAKE, FAKE + 8, need, None, None) == B.INVALID_ARG   # misaligned
    assert b"aligned" in lib.kvpop_last_error()
    # T = 0 needs no workspace and enqueues nothing
    assert F(FAKE, FAKE, _cu(0, 0), B.Shape(1, 0, 4, 2, 128), 0.1, 4, FAKE, FAKE, None, 0, None, None) == B.OK


def test_target_workspace_bytes(lib):
    # 16 bytes of normaliser row per (query head, token), rounded up to 256
    r = lambda x: (x + 255) // 256 * 256
    assert lib.kvpop_target_workspace_bytes(B.Shape(1, 16384, 32, 8, 128)) == 32 * 16384 * 16
    assert lib.kvpop_target_workspace_bytes(B.Shape(3, 101, 4, 2, 64)) == r(4 * 101 * 16)
    assert lib.kvpop_target_workspace_bytes(B.Shape(1, 0, 4, 2, 64)) == 0


def test_keep_mask_rejects(lib):
    cu, sh = _cu(0, 100), _shape()
    bud = _cu(50)
    assert lib.kvpop_keep_mask(None, cu, sh, 16, 4, bud, FAKE, None) == B.INVALID_ARG
    assert lib.kvpop_keep_mask(FAKE, cu, sh, 16, 4, None, FAKE, None) == B.INVALID_ARG
    assert lib.kvpop_keep_mask(FAKE, cu, sh, 16, 4, _cu(19), FAKE, None) == B.INVALID_ARG   # < sinks + window
    assert lib.kvpop_keep_mask(FAKE, cu, sh, -1, 4, bud, FAKE, None) == B.INVALID_ARG
    assert lib.kvpop_keep_mask(FAKE, cu, sh, 16, -4, bud, FAKE, None) == B.INVALID_ARG


def test_thresholds_reject(lib):
    cu, sh = _cu(0, 100), _shape()
    bud = _cu(50)
    T = lib.kvpop_prefix_topk_thresholds
    assert T(None, cu, sh, 16, 4, bud, FAKE, FAKE, None) == B.INVALID_ARG
    assert T(FAKE, cu, sh, 16, 4, bud, None, FAKE, None) == B.INVALID_ARG
    assert T(FAKE, cu, sh, 16, 4, bud, FAKE, None, None) == B.INVALID_ARG
    assert T(FAKE, cu, sh, 16, 4, None, FAKE, FAKE, None) == B.INVALID_ARG
    assert T(FAKE, cu, sh, 16, 4, _cu(19), FAKE, FAKE, None) == B.INVALID_ARG        # below sinks + window
    assert T(FAKE, _cu(0, 0), B.Shape(1, 0, 4, 2, 128), 16, 4, bud, FAKE, FAKE, None) == B.OK


def test_static_cache_rejects(lib):
    cu, sh = _cu(0, 100), _shape()
    C = lib.kvpop_compact_kv
    assert C(None, FAKE, FAKE, cu, sh, 8, FAKE, FAKE, FAKE, FAKE, None) == B.INVALID_ARG
    assert C(FAKE, FAKE, FAKE, cu, sh, 0, FAKE, FAKE, FAKE, FAKE, None) == B.INVALID_ARG          # capacity
    assert C(FAKE, FAKE + 8, FAKE, cu, sh, 8, FAKE, FAKE, FAKE, FAKE, None) == B.INVALID_ARG      # alignment
    assert C(FAKE, FAKE, FAKE, cu, _shape(d=96), 8, FAKE, FAKE, FAKE, FAKE, None) == B.UNSUPPORTED
    cs = B.CacheShape(1, 8, 2, 128, 1000)
    need = lib.kvpop_decode_workspace_bytes(cs)
    assert need == 1 * 8 * 8 * 130 * 4                                                             # 8 splits of 128 slots
    assert lib.kvpop_decode_workspace_bytes(B.CacheShape(1, 6, 2, 128, 10)) == 0                    # group of 3
    D = lib.kvpop_decode_attention
    assert D(FAKE, FAKE, FAKE, FAKE, cs, 0.1, FAKE, None, FAKE, need - 1, None) == B.INVALID_ARG   # workspace
    assert D(FAKE, FAKE, FAKE, FAKE, cs, 0.0, FAKE, None, FAKE, need, None) == B.INVALID_ARG       # scale
    assert D(FAKE, FAKE, FAKE, None, cs, 0.1, FAKE, None, FAKE, need, None) == B.INVALID_ARG       # count
    assert D(FAKE + 8, FAKE, FAKE, FAKE, cs, 0.1, FAKE, None, FAKE, need, None) == B.INVALID_ARG   # q alignment
    assert D(FAKE, FAKE, FAKE, FAKE, B.CacheShape(1, 64, 2, 128, 10), 0.1, FAKE, None, FAKE, need,
             None) == B.UNSUPPORTED                                                                # group of 32
    N = lib.kvpop_decode_attention_noalloc
    assert N(FAKE, FAKE, FAKE, None, cs, 0.1, FAKE, None, None) == B.INVALID_ARG
    assert N(FAKE, FAKE, FAKE, FAKE, cs, -1.0, FAKE, None, None) == B.INVALID_ARG
    big = B.CacheShape(64, 64, 8, 128, 8192)                                                       # 68 MB of partials
    assert N(FAKE, FAKE, FAKE, FAKE, big, 0.1, FAKE, None, None) == B.UNSUPPORTED
    assert b"fixed scratch" in lib.kvpop_last_error()


def test_pipeline_rejects(lib):
    cu, sh = _cu(0, 100), _shape()
    bud = _cu(50)
    tneed = lib.kvpop_target_workspace_bytes(sh)
    P = lib.kvpop_future_targets
    assert P(FAKE, FAKE, cu, sh, 0.1, 16, 4, _cu(10), FAKE, FAKE, FAKE, FAKE, tneed, None, None) == B.INVALID_ARG
    assert P(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, FAKE, FAKE, tneed - 16, None, None) == B.INVALID_ARG
    assert P(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, FAKE, FAKE + 4, tneed, None, None) == B.INVALID_ARG
    assert P(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, None, FAKE, tneed, None, None) == B.INVALID_ARG
    need = lib.kvpop_host_workspace_bytes(sh)
    assert lib.kvpop_future_targets_host(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, FAKE, need - 1, None,
                                         None) == B.INVALID_ARG
    assert lib.kvpop_future_targets_host(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, FAKE + 16, need, None,
                                         None) == B.INVALID_ARG
    F = lib.kvpop_future_targets_fused
    fneed = lib.kvpop_fused_workspace_bytes(cu, sh)
    assert F(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, FAKE, None, fneed, None, None) == B.INVALID_ARG
    assert F(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, FAKE, FAKE, fneed - 1, None, None) == B.INVALID_ARG
    assert F(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, FAKE, FAKE + 2, fneed, None, None) == B.INVALID_ARG
    assert F(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, FAKE, FAKE, FAKE, FAKE + 4, fneed, None, None) == B.INVALID_ARG
    assert F(FAKE, FAKE, cu, sh, 0.1, 16, 4, _cu(10), FAKE, FAKE, FAKE, FAKE, fneed, None, None) == B.INVALID_ARG
    assert F(FAKE, FAKE, cu, sh, 0.1, 16, 4, bud, None, FAKE, FAKE, FAKE, fneed, None, None) == B.INVALID_ARG
    assert lib.kvpop_check_device_status(None, None) == B.INVALID_ARG
    assert lib.kvpop_selftest_bounded_wait(FAKE, 0, None) == B.INVALID_ARG
    assert lib.kvpop_selftest_bounded_wait(None, 1000, None) == B.INVALID_ARG


def test_workspace_bytes(lib):
    sh = B.Shape(1, 16384, 32, 8, 128)
    r = lambda x: (x + 255) // 256 * 256
    T = 16384
    # q, k, lse, target, keep, then for the largest KV-head group (eight groups
    # of one head) the normaliser rows (G = 4 query heads x T x 16 bytes) and
    # the split partials (4 query heads x 4 column groups x T floats)
    want = (r(T * 32 * 128 * 2) + r(T * 8 * 128 * 2) + r(T * 32 * 4) + r(T * 8 * 4) + r(T * 8) +
            r(4 * 1 * T * 16) + r(4 * 1 * 4 * T * 4))
    assert lib.kvpop_host_workspace_bytes(sh) == want
    assert lib.kvpop_host_workspace_bytes(B.Shape(1, 0, 32, 8, 128)) == 0


def test_split_target_rejects_and_sizes(lib):
    cu, sh = _cu(0, 100), _shape()                       # 4 query heads over 2 KV heads
    need = lib.kvpop_target_split_workspace_bytes(sh)
    # normaliser rows (query heads x T x 16 bytes, rounded up to 256), then
    # query heads x column groups x T floats
    assert need == 6400 + 4 * 4 * 100 * 4
    S = lib.kvpop_future_target_split
    assert S(FAKE, FAKE, cu, sh, 0.1, 16, FAKE, FAKE, None, need, None, None) == B.INVALID_ARG       # no workspace
    assert S(FAKE, FAKE, cu, sh, 0.1, 16, FAKE, FAKE, FAKE, need - 4, None, None) == B.INVALID_ARG   # too small
    assert S(FAKE, FAKE, cu, sh, 0.1, 16, FAKE, FAKE, FAKE + 4, need, None, None) == B.INVALID_ARG   # misaligned
    assert S(FAKE, FAKE, cu, sh, 0.1, -1, FAKE, FAKE, FAKE, need, None, None) == B.INVALID_ARG       # window
    assert S(FAKE, FAKE, cu, sh, 0.1, 16, None, FAKE, FAKE, need, None, None) == B.INVALID_ARG       # lse
    assert lib.kvpop_target_split_workspace_bytes(B.Shape(1, 100, 6, 4, 128)) == 0                  # 6 % 4 != 0


def test_fused_workspace_bytes(lib):
    # one int32 per (query head, 128-row tile of each sequence), plus two
    # completion counters, rounded up to 256; then 16 bytes of normaliser row
    # per (query head, token)
    r = lambda x: (x + 255) // 256 * 256
    assert lib.kvpop_fused_workspace_bytes(_cu(0, 16384), B.Shape(1, 16384, 32, 8, 128)) == \
        r((32 * 128 + 2) * 4) + 32 * 16384 * 16
    assert lib.kvpop_fused_workspace_bytes(_cu(0, 1, 129, 129, 300), B.Shape(4, 300, 4, 2, 64)) == \
        r((4 * (1 + 1 + 0 + 2) + 2) * 4) + r(4 * 300 * 16)
    assert lib.kvpop_fused_workspace_bytes(None, B.Shape(1, 10, 4, 2, 64)) == 0
    assert lib.kvpop_fused_workspace_bytes(_cu(0, 10), B.Shape(1, 10, 0, 2, 64)) == 0


def test_empty_input_is_a_no_op(lib):
    # T = 0: valid, nothing to enqueue, no device call.
    assert lib.kvpop_row_lse(FAKE, FAKE, _cu(0, 0), B.Shape(1, 0, 4, 2, 128), 0.1, FAKE, None, None) == B.OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(B, "_handle", None)
    with pytest.raises(RuntimeError, match="missing"):
        B.lib()

"""The FMA-pipe exp2 of the attention kernels, checked on the CPU.

The softmax passes evaluate part of their exponentials as 2^y = 2^n * p(f)
(Cody-Waite reduction, a minimax polynomial with p(0) = 1, the exponent
added as an integer): degree 4 in the row-logsumexp pass (kP1..kP4), degree
3 in the transposed pass (kT1..kT3).  These tests pin the kernel's
coefficients to the Remez fits that produce them and bound the relative
error of the whole construction, emulated step by step in float32, against
2^y in float64.
"""
import importlib.util
import pathlib
import re

import numpy as np
import pytest

CSRC = pathlib.Path(__file__).resolve().parents[1] / "future_attention_targets_b200" / "csrc"
# degree -> (kernel constant prefix, minimax bound, bound with float32 rounding of the steps)
SETS = {4: ("kP", 2.9e-6, 3.5e-6), 3: ("kT", 8.6e-5, 9e-5)}


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", CSRC / "fit_exp2_poly.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coefficients(degree):
    prefix = SETS[degree][0]
    src = (CSRC / "attn_kernels.cu").read_text()
    pat = "constexpr float " + ", ".join(f"{prefix}{k} = ([0-9a-fx.p+-]+)f" for k in range(1, degree + 1)) + ";"
    m = re.search(pat, src)
    assert m, f"{prefix}1..{prefix}{degree} not found in attn_kernels.cu"
    return np.array([float.fromhex(x) for x in m.groups()], dtype=np.float32)


@pytest.mark.parametrize("degree", [4, 3])
def test_kernel_coefficients_are_the_fit(degree):
    fit = _fit_module()
    c, err = fit.remez(degree)
    np.testing.assert_array_equal(c.astype(np.float32), _kernel_coefficients(degree))
    assert err < SETS[degree][1]
    assert fit.fp32_horner_error(_kernel_coefficients(degree)) < SETS[degree][2]


def _emulated_exp2(y, coeffs, hi=None):
    """The kernel's steps in float32: clamp (below at -126; above at `hi` where the
    kernel clamps there too), n = floor(y) (what adding 1.5 * 2^23 rounded toward
    minus infinity leaves), f = y - n, Horner from the highest coefficient down to
    the pinned 1, then n added to the exponent bits."""
    y = np.maximum(y.astype(np.float32), np.float32(-126.0))
    if hi is not None:
        y = np.minimum(y, np.float32(hi))
    n = np.floor(y).astype(np.float32)
    f = (y - n).astype(np.float32)
    q = np.full_like(f, coeffs[-1])
    for ck in coeffs[-2::-1]:
        q = (q * f + ck).astype(np.float32)
    q = (q * f + np.float32(1.0)).astype(np.float32)
    bits = q.view(np.uint32).astype(np.int64) + (n.astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)   # the 32-bit add wraps


@pytest.mark.parametrize("degree", [4, 3])
def test_emulated_exp2_error_bound(degree):
    coeffs = _kernel_coefficients(degree)
    rng = np.random.default_rng(7)
    y = np.concatenate([rng.uniform(-126.0, 0.0, 400_000), rng.uniform(-1.0, 0.0, 100_000)]).astype(np.float32)
    rel = np.abs(_emulated_exp2(y, coeffs).astype(np.float64) / np.exp2(y.astype(np.float64)) - 1.0)
    assert float(rel.max()) < SETS[degree][2]
    # integers are exact: p(0) = 1
    k = -np.arange(0, 127, dtype=np.float32)
    np.testing.assert_array_equal(_emulated_exp2(k, coeffs), np.exp2(k.astype(np.float64)).astype(np.float32))


@pytest.mark.parametrize("degree", [4, 3])
def test_large_arguments_need_the_upper_clamp(degree):
    """Above 127 the exponent add wraps: without the upper clamp 2^y of a large argument comes out tiny
    (so a tile's sum would silently lose its largest terms); with it the result is at least 2^127, so the
    sum reaches the row logsumexp's overflow check."""
    coeffs = _kernel_coefficients(degree)
    y = np.linspace(128.0, 300.0, 2000, dtype=np.float32)
    wrapped = _emulated_exp2(y, coeffs)
    with np.errstate(invalid="ignore"):   # some wrapped bit patterns are NaNs
        reaches_check = np.isfinite(wrapped) & (np.abs(wrapped) >= np.float32(2.0 ** 64))
    assert np.mean(reaches_check) < 0.5
    clamped = _emulated_exp2(y, coeffs, hi=127.0).astype(np.float64)
    assert np.all(np.isfinite(clamped)) and np.all(clamped >= 2.0 ** 127)
    # below the clamp nothing changes
    z = np.linspace(-126.0, 127.0, 5000, dtype=np.float32)
    np.testing.assert_array_equal(_emulated_exp2(z, coeffs, hi=127.0), _emulated_exp2(z, coeffs))

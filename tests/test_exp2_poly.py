"""The FP32-pipe exp2 of the scan kernels' general-A path (scan.cuh, exp2_fma2): its constants
are the fit that fit_exp2.py computes, and the method -- reduction to the nearest integer by the
1.5 * 2^23 shift, the degree-5 polynomial in fp32 Horner steps, the exponent-field scaling, the
clamp to [-125, 127] -- stays within its stated bounds of 2^x, with no bias near x = 0.  The method is emulated here in
numpy with fp32 rounding after every step; the kernels' use of it is covered by the GPU parity
tests of the general-A path."""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_state_space_46_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2", os.path.join(CSRC, "fit_exp2.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_constants():
    text = open(os.path.join(CSRC, "scan.cuh")).read()
    found = dict(re.findall(r"constexpr float kExp2C(\d) = ([0-9.eE+-]+)f;", text))
    return np.array([np.float32(float(found[str(k)])) for k in range(len(found))], dtype=np.float32)


def _f32(v):
    return np.asarray(v, dtype=np.float64).astype(np.float32)


def emulate(x, c):
    """exp2_fma2 step by step; every arithmetic result rounded to fp32 as the FP32 pipe does
    (a fused multiply-add: the exact product and sum in fp64, then one rounding)."""
    shift = np.float32(12582912.0)
    xc = np.minimum(np.maximum(_f32(x), np.float32(-125.0)), np.float32(127.0))
    t = _f32(xc.astype(np.float64) + np.float64(shift))
    j = _f32(t.astype(np.float64) - np.float64(shift))
    f = _f32(xc.astype(np.float64) - j.astype(np.float64))
    p = _f32(c[5].astype(np.float64) * f + c[4])
    for k in (3, 2, 1, 0):
        p = _f32(p.astype(np.float64) * f + c[k])
    jint = t.view(np.int32) - shift.view(np.int32)
    r = (p.view(np.int32) + (jint << 23)).view(np.float32)
    xs = _f32(x)
    return np.where(np.isnan(xs), xs, r)


def test_constants_are_the_fit():
    fitted = _fit_module().fit()
    assert np.array_equal(_header_constants(), fitted)


def test_reduction_is_exact_and_in_range():
    x = _f32(np.linspace(-125.0, 127.0, 400001))
    shift = np.float32(12582912.0)
    t = _f32(x.astype(np.float64) + shift)
    j = _f32(t.astype(np.float64) - shift)
    f = _f32(x.astype(np.float64) - j)
    assert np.all(np.abs(f) <= 0.5)
    assert np.array_equal(j, np.round(j)) and np.all(np.abs(j.astype(np.float64) - x) <= 0.5)
    assert np.array_equal(f.astype(np.float64) + j.astype(np.float64), x.astype(np.float64))
    assert np.array_equal(t.view(np.int32) - shift.view(np.int32), j.astype(np.int32))


@pytest.mark.parametrize("lo,hi", [(-0.5, 0.5), (-30.0, 0.0), (-125.0, -100.0), (0.0, 127.0)])
def test_relative_error_bound(lo, hi):
    c = _header_constants()
    x = _f32(np.linspace(lo, hi, 300001))
    got = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() <= 1.7e-7, rel.max()


def test_no_bias_near_one():
    """Decay factors close to 1 are the ones whose errors compound over many steps: the
    constant term is exactly 1, and the signed error there averages out to rounding noise."""
    c = _header_constants()
    assert c[0] == np.float32(1.0)
    x = _f32(np.linspace(-0.02, 0.02, 200001))
    got = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    signed = (got - ref) / ref
    assert abs(signed.mean()) < 2e-9 and np.abs(signed).max() < 7e-8


def test_clamped_inputs():
    c = _header_constants()
    x = _f32([-1e30, -1000.0, -126.0, -125.0, 127.0, 128.0, 1e30])
    got = emulate(x, c).astype(np.float64)
    low = np.exp2(-125.0)
    assert np.all(got[:4] > 0) and np.allclose(got[:4], low, rtol=2e-7)
    assert np.allclose(got[4:], np.exp2(127.0), rtol=2e-7) and np.all(np.isfinite(got))


def test_nan_propagates():
    c = _header_constants()
    got = emulate(_f32([np.nan, -1.0, np.nan]), c)
    assert np.isnan(got[0]) and np.isnan(got[2]) and np.isfinite(got[1])

"""The kernels' FMA-pipe exp2 (ex2_fma in csrc/tc_common.cuh): its constants are
the ones the fitting script produces, and its fp32 algorithm (round-to-nearest
split via 1.5 * 2^23, cubic for 2^f, exponent-field add) stays within its
error bound against exp2 over the range the kernels use."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "random_feature_linear_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    src = open(os.path.join(CSRC, "tc_common.cuh")).read()
    body = src[src.index("float ex2_fma("):]
    body = body[:body.index("return")]
    nums = [float(x) for x in re.findall(r"(\d\.\d+)f", body)]
    # fmaf(fmaf(fmaf(c3, f, c2), f, c1), f, c0)
    return [nums[3], nums[2], nums[1], nums[0]]


def ex2_fma_emulated(x):
    f32 = np.float32
    x = np.minimum(np.maximum(x.astype(f32), f32(-126)), f32(128))
    big = f32(12582912.0)
    t = (x + big).astype(f32)
    f = (x - (t - big).astype(f32)).astype(f32)
    c0, c1, c2, c3 = (f32(c) for c in _header_coefficients())
    # fmaf rounds once; emulate with float64 products rounded to fp32
    p = (c3.astype(np.float64) * f + c2).astype(f32)
    p = (p.astype(np.float64) * f + c1).astype(f32)
    p = (p.astype(np.float64) * f + c0).astype(f32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_constants_match_fit():
    mod = _fit_module()
    np.testing.assert_allclose(_header_coefficients(), mod.coefficients_f32(), rtol=1e-7)
    _, err = mod.fit()
    assert err < 1e-4


def test_error_bound_over_kernel_range():
    x = np.linspace(-125.0, 127.0, 2_000_003).astype(np.float32)
    got = ex2_fma_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1.2e-4, rel.max()


def test_clamping():
    x = np.array([-1000.0, -126.0, 128.5, 200.0], np.float32)
    y = ex2_fma_emulated(x)
    assert y[0] == y[1] and 0 < y[0] < 1e-37
    assert y[2] == y[3] and y[2] > 3.4e38

"""The polynomial exponential of the attention softmax, pinned on the CPU.

The kernel constants (exp2_poly.cuh) must be exactly what the committed fit
(csrc/exp2_poly_fit.py: Lawson's minimax iteration on Chebyshev nodes) produces
when rounded to fp32, and that polynomial must meet the stated bound: relative
error <= 7.5e-5 for 2^f on [-1/2, 1/2], hence for 2^x after the range reduction
2^x = 2^j 2^f.  The bound is checked against numpy's exp2 in fp64, and the
range-reduced evaluation is emulated in fp32 over the softmax's input range.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "patch_diffusion_unet_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_coefficients():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    body = text[text.index("ex2_poly_pair_f32"):]
    vals = re.findall(r"f2\(([0-9.]+)f, \1f\)", body)
    # f^3 and f^2 in the first fma, then f, then the constant term
    return [float(np.float32(v)) for v in vals if v not in ("12582912.", "-1.")][:4]


def test_kernel_constants_are_the_committed_fit():
    m = _fit_module()
    assert _kernel_coefficients() == m.fp32_coefficients()


def test_fit_meets_the_stated_bound():
    m = _fit_module()
    c = m.fp32_coefficients()
    err = m.max_rel_error(c)
    assert err <= 7.5e-5
    # equioscillation: a minimax fit of degree 3 touches its maximum error at 5 points
    f = np.linspace(-0.5, 0.5, 200001)
    r = np.polyval(c, f) / 2.0 ** f - 1.0
    ext = [i for i in range(1, len(f) - 1) if abs(r[i]) >= abs(r[i - 1]) and abs(r[i]) >= abs(r[i + 1])]
    ext = [i for i in [0] + ext + [len(f) - 1] if abs(r[i]) > 0.95 * err]
    assert len(ext) >= 5
    # a plain Taylor cubic is ten times worse: the fit is doing something
    taylor = [np.log(2) ** 3 / 6, np.log(2) ** 2 / 2, np.log(2), 1.0]
    assert m.max_rel_error(taylor) > 5 * err


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def emulate_fp32(x):
    """The kernel's steps in fp32 (fma as fp64 product-sum rounded once)."""
    c3, c2, c1, c0 = (np.float32(v) for v in _kernel_coefficients())
    x = np.maximum(np.float32(x), np.float32(-125.0)).astype(np.float32)
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = _fma32(j, np.float32(-1.0), x)
    p = _fma32(c3, f, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_range_reduced_evaluation_in_fp32():
    x = np.concatenate([np.linspace(-125.0, 0.0, 400001), -np.arange(0, 125) - 0.5, [0.0, -0.5, 0.5, -125.0]])
    x = x.astype(np.float32)
    y = emulate_fp32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(y / want - 1.0)
    assert rel.max() <= 7.5e-5 + 4 * 2.0 ** -24
    # below the clamp the value is 2^-125 (within the bound): negligible next to a row maximum of 1
    assert abs(float(emulate_fp32(np.float32(-300.0))) / 2.0 ** -125 - 1.0) <= 7.5e-5

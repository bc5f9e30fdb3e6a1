"""The scan kernels' softplus polynomial on the host (no GPU).

* The coefficients written in ss2d_kernels.cuh are, as float32 values, the
  ones csrc/fit_softplus.py produces (its least-squares fit of log1p(e)/e).
* Evaluated the way the kernel evaluates it (float32 Horner steps with one
  rounding each, e = exp(-|z|) rounded to float32, final fmaf with
  max(z, 0)), softplus stays within 4e-7 relative error of float64
  log1p(exp(z)) over z in [-40, 40].  The kernel's e comes from the
  multi-function unit's exp2 instead; its own error adds to this and is
  bounded on the GPU by tests/test_gpu_long_fp32.py.
"""
from __future__ import annotations

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_scan_ss2d_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_softplus",
                                                  os.path.join(CSRC, "fit_softplus.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def kernel_coefficients() -> np.ndarray:
    """The Horner coefficients of softplus_f, highest degree first."""
    src = open(os.path.join(CSRC, "ss2d_kernels.cuh")).read()
    body = src[src.index("float softplus_f(float z)"):]
    body = body[:body.index("}")]
    first = re.search(r"float q = ([-+0-9.e]+)f;", body).group(1)
    rest = re.findall(r"q = fmaf\(q, e, ([-+0-9.e]+)f\);", body)
    return np.array([float(first)] + [float(c) for c in rest])


def f32_fma(a, b, c):
    """fmaf emulated: the float32 product is exact in float64; one rounding
    of the float64 sum to float32 (double rounding can differ from a true
    fmaf by one ulp in rare halfway cases, far below the bound)."""
    return (np.float64(a) * np.float64(b) + np.float64(c)).astype(np.float32)


def softplus_like_kernel(z: np.ndarray, coef: np.ndarray) -> np.ndarray:
    z = z.astype(np.float32)
    e = np.exp(-np.abs(z.astype(np.float64))).astype(np.float32)
    c32 = coef.astype(np.float32)
    q = np.full_like(z, c32[0])
    for c in c32[1:]:
        q = f32_fma(q, e, np.full_like(z, c))
    return f32_fma(e, q, np.maximum(z, np.float32(0)))


def test_kernel_coefficients_are_the_fit():
    fit = _fit_module().fit()
    got = kernel_coefficients()
    assert got.shape == fit.shape == (8,)
    assert np.array_equal(got.astype(np.float32), fit.astype(np.float32))


def test_fit_error_in_float64():
    mod = _fit_module()
    assert mod.max_rel_error(mod.fit()) < 2.5e-7


def test_float32_evaluation_bound():
    z = np.linspace(-40.0, 40.0, 400001)
    got = softplus_like_kernel(z, kernel_coefficients()).astype(np.float64)
    zz = z.astype(np.float32).astype(np.float64)   # the value the kernel sees
    want = np.maximum(zz, 0) + np.log1p(np.exp(-np.abs(zz)))
    rel = np.abs(got - want) / want
    assert rel.max() <= 4e-7, f"max relative error {rel.max():.3e} at z = {z[rel.argmax()]}"

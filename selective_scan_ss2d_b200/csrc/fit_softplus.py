"""Produce the polynomial behind the scan kernels' softplus (``softplus_f`` in
ss2d_kernels.cuh and ss2d_backward.cuh).

softplus(z) = log(1 + e^z) = max(z, 0) + log1p(e), with e = exp(-|z|) in
(0, 1].  The kernels evaluate log1p(e) = e * q(e), q a degree-7 polynomial
that approximates log1p(e) / e on [0, 1] (the limit at e = 0 is 1).  The
coefficients are the ordinary least-squares fit of that function on the 256
Chebyshev nodes of the first kind mapped to [0, 1]; nothing else goes into
them.

    python selective_scan_ss2d_b200/csrc/fit_softplus.py

prints them highest degree first, in the order the kernels' Horner loop uses,
with ten significant digits (the digits the kernels hold), and the largest
relative error of e * q(e) against log1p(e) on a fine grid, evaluated in
float64.
"""
from __future__ import annotations

import numpy as np

DEGREE = 7
NODES = 256


def target(e: np.ndarray) -> np.ndarray:
    """log1p(e) / e, with its limit 1 at e = 0."""
    e = np.asarray(e, dtype=np.float64)
    out = np.ones_like(e)
    nz = e != 0
    out[nz] = np.log1p(e[nz]) / e[nz]
    return out


def fit(degree: int = DEGREE, nodes: int = NODES) -> np.ndarray:
    """Least-squares coefficients, highest degree first."""
    k = np.arange(nodes)
    e = 0.5 - 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))
    V = np.vander(e, degree + 1)
    coef, *_ = np.linalg.lstsq(V, target(e), rcond=None)
    return coef


def max_rel_error(coef: np.ndarray, samples: int = 200001) -> float:
    e = np.linspace(0.0, 1.0, samples)[1:]
    approx = e * np.polyval(coef, e)
    return float(np.max(np.abs(approx - np.log1p(e)) / np.log1p(e)))


def main() -> None:
    coef = fit()
    for c in coef:
        print(f"{c:.9e}")
    print(f"max relative error of e*q(e) (float64): {max_rel_error(coef):.3e}")


if __name__ == "__main__":
    main()

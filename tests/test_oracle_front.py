"""Pins of the float64 front oracle (``oracle/ss2d_front_np.py``): the causal
depthwise conv1d + SiLU + x_proj + dt_proj of the tutorial's SelectiveSSM
that feeds the scan.

* the conv against NumPy's own ``convolve`` (a library routine) per channel,
  its impulse response (the taps, last tap first) and its causality;
* x_proj against selector weights (rows that pick one channel), and
  linearity in x_proj's weight;
* the split into (dt_raw, B, C) and dt_proj's product;
* planted mistakes in the oracle's source, each caught by one of these.
"""
from __future__ import annotations

import inspect
import types

import numpy as np
import pytest

from oracle import ss2d_front_np
from oracle.ss2d_oracle_np import silu


def _problem(seed, B=2, L=11, D=5, N=3, kc=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, L, D)), rng.standard_normal((D, kc)),
            rng.standard_normal(D), rng.standard_normal((1 + 2 * N, D)),
            rng.standard_normal(D))


def check_conv_against_numpy(mod):
    x, w, b, _, _ = _problem(1)
    got = mod.causal_depthwise_conv(x, w, b)
    L = x.shape[1]
    for bb in range(x.shape[0]):
        for d in range(x.shape[2]):
            # the layer correlates: reversed taps with numpy's convolution,
            # the first L outputs of the full convolution
            want = np.convolve(x[bb, :, d], w[d, ::-1])[:L] + b[d]
            np.testing.assert_allclose(got[bb, :, d], want, rtol=1e-13, atol=1e-13)


def check_impulse_and_causality(mod):
    _, w, b, _, _ = _problem(2)
    D, kc = w.shape
    L, l0 = 12, 5
    x = np.zeros((1, L, D))
    x[0, l0, :] = 1.0
    c = mod.causal_depthwise_conv(x, w, b)
    for i in range(kc):   # output l0 + i sees the impulse through tap kc-1-i
        np.testing.assert_allclose(c[0, l0 + i], w[:, kc - 1 - i] + b, rtol=1e-14)
    np.testing.assert_allclose(c[0, :l0], np.broadcast_to(b, (l0, D)), rtol=1e-14)
    np.testing.assert_allclose(c[0, l0 + kc:], np.broadcast_to(b, (L - l0 - kc, D)),
                               rtol=1e-14)


def check_projections(mod):
    x, w, b, W_x, w_dt = _problem(3)
    D = x.shape[2]
    N = (W_x.shape[0] - 1) // 2
    u, delta, Bs, Cs = mod.front(x, w, b, W_x, w_dt)
    ref_u = silu(mod.causal_depthwise_conv(x, w, b))            # (B, L, D)
    np.testing.assert_allclose(u, ref_u.transpose(0, 2, 1), rtol=1e-13)
    # selector weights: row r picks channel sel[r], so x_proj returns u itself
    sel = np.arange(1 + 2 * N) % D
    P = np.zeros_like(W_x)
    P[np.arange(1 + 2 * N), sel] = 1.0
    u2, delta2, B2, C2 = mod.front(x, w, b, P, np.ones(D))
    np.testing.assert_allclose(delta2[:, 0], np.broadcast_to(
        ref_u[:, :, sel[0]][:, None, :], delta2[:, 0].shape), rtol=1e-13)
    for n in range(N):
        np.testing.assert_allclose(B2[:, 0, n], ref_u[:, :, sel[1 + n]], rtol=1e-13)
        np.testing.assert_allclose(C2[:, 0, n], ref_u[:, :, sel[1 + N + n]], rtol=1e-13)
    # dt_proj: delta[d] = w_dt[d] * dt_raw, dt_raw the first output of x_proj
    dt_raw = ref_u @ W_x[0]
    np.testing.assert_allclose(delta[:, 0], w_dt[None, :, None] * dt_raw[:, None, :],
                               rtol=1e-12, atol=1e-13)
    # linear in the x_proj weight
    W2 = np.random.default_rng(4).standard_normal(W_x.shape)
    _, d_a, B_a, C_a = mod.front(x, w, b, W_x + 2.0 * W2, w_dt)
    _, d_b, B_b, C_b = mod.front(x, w, b, W2, w_dt)
    np.testing.assert_allclose(B_a, Bs + 2.0 * B_b, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(C_a, Cs + 2.0 * C_b, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(d_a, delta + 2.0 * d_b, rtol=1e-12, atol=1e-12)


CHECKS = [check_conv_against_numpy, check_impulse_and_causality, check_projections]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_front_pin(check):
    check(ss2d_front_np)


MUTATIONS = {
    "conv_not_causal": ("src = l - (kc - 1) + j", "src = l - (kc - 1) // 2 + j"),
    "conv_taps_reversed": ("acc = acc + w[None, :, j] * x[:, src, :]",
                           "acc = acc + w[None, :, kc - 1 - j] * x[:, src, :]"),
    "conv_bias_dropped": ("acc = np.array(bias, dtype=np.float64)[None, :].repeat(Bb, axis=0)",
                          "acc = np.zeros((Bb, D))"),
    "silu_dropped": ("u_bld = silu(causal_depthwise_conv(x, conv_w, conv_b))",
                     "u_bld = causal_depthwise_conv(x, conv_w, conv_b)"),
    "B_and_C_swapped": ("Bm = x_dbl[:, :, 1:1 + N]", "Bm = x_dbl[:, :, 1 + N:1 + 2 * N]"),
    "dt_proj_weight_dropped": (
        "delta = np.asarray(w_dt, dtype=np.float64)[None, :, None] * dt_raw[:, None, :]",
        "delta = np.ones_like(np.asarray(w_dt))[None, :, None] * dt_raw[:, None, :]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_front_mistake_is_caught(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(ss2d_front_np)
    assert src.count(old) == 1, name
    src = src.replace(old, new).replace("from .ss2d_oracle_np import",
                                        "from oracle.ss2d_oracle_np import")
    mod = types.ModuleType(f"front_mutant_{name}")
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    caught = []
    for check in CHECKS:
        try:
            check(mod)
        except Exception:   # a failed pin, or a mistake that breaks the code outright
            caught.append(check.__name__)
    assert caught, f"planted mistake '{name}' passed every pin"

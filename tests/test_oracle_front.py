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
import os
import types

import numpy as np
import pytest

import oracle
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


# ---------------------------------------------------------------------------
# the per-direction front (Vim block) and its precision readings
# ---------------------------------------------------------------------------
def _problem_k(seed, B=2, L=10, D=6, N=3, K=2, kc=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, L, D)), rng.standard_normal((K, D, kc)),
            rng.standard_normal((K, D)), rng.standard_normal((K, 1 + 2 * N, D)) / np.sqrt(D),
            rng.standard_normal((K, D)))


def check_directions_against_front(mod):
    """Direction 0 is the one-direction front of the sequence, direction 1
    the one-direction front of the sequence reversed along L."""
    x, w, b, W_x, w_dt = _problem_k(5)
    got = mod.front_directions(x, w, b, W_x, w_dt)
    for k, seq in ((0, x), (1, x[:, ::-1, :])):
        want = mod.front(seq, w[k], b[k], W_x[k], w_dt[k])
        for g, wt in zip(got, want):   # front's u has no direction axis
            np.testing.assert_allclose(g[:, k], wt if wt.ndim == 3 else wt[:, 0],
                                       rtol=1e-13, atol=1e-14)


def check_bf16_rounding_golden(mod):
    """round_storage("bf16") against the hand-worked table of
    tests/golden/bf16_rne.txt (float32 pattern -> bfloat16 pattern)."""
    path = os.path.join(os.path.dirname(__file__), "golden", "bf16_rne.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    f32 = np.array([int(r[0], 16) for r in rows], dtype=np.uint32).view(np.float32)
    want = (np.array([int(r[1], 16) for r in rows], dtype=np.uint32) << 16).view(np.float32)
    got = mod.round_storage(f32.astype(np.float64), "bf16")
    np.testing.assert_array_equal(got, want.astype(np.float64))


def check_operand_rounding(mod):
    """bf16 operands: exact when u and W_x are bf16 values already; otherwise
    within the rounding bound of the two operands (2^-8 relative each
    product, taken over |u| |W|)."""
    x, w, b, W_x, w_dt = _problem_k(6, K=1)
    exact = mod.front_directions(x, w, b, W_x, w_dt)
    rounded = mod.front_directions(x, w, b, W_x, w_dt, operand="bf16")
    u = mod.silu(mod.causal_depthwise_conv(x, w[0], b[0]))          # (B, L, D)
    bound = (np.abs(u) @ np.abs(W_x[0]).T) * (2.0 ** -8 + 2.0 ** -16)   # (B, L, 1 + 2N)
    N = (W_x.shape[1] - 1) // 2
    np.testing.assert_array_less(np.abs(rounded[2][:, 0] - exact[2][:, 0]),
                                 bound[:, :, 1:1 + N].transpose(0, 2, 1) + 1e-300)
    assert np.abs(rounded[2] - exact[2]).max() > 0   # the rounding is applied
    # bf16-exact operands: W_x of small dyadic values, a conv whose SiLU output
    # is 0 (zero taps and a large negative bias give u = -0 to double precision)
    W2 = np.round(W_x * 8) / 8
    w0, b0 = np.zeros_like(w), np.full_like(b, -800.0)
    a = mod.front_directions(x, w0, b0, W2, w_dt)
    r = mod.front_directions(x, w0, b0, W2, w_dt, operand="bf16")
    for g, h in zip(a, r):
        np.testing.assert_array_equal(g, h)


def check_storage(mod):
    """u as stored: each storage dtype's rounding of the exact u (the scan's
    input), the projections untouched by it."""
    x, w, b, W_x, w_dt = _problem_k(7)
    exact = mod.front_directions(x, w, b, W_x, w_dt)
    for st, cast in (("f32", np.float32), ("f16", np.float16)):
        got = mod.front_directions(x, w, b, W_x, w_dt, storage=st)
        np.testing.assert_array_equal(got[0], exact[0].astype(cast).astype(np.float64))
        for g, e in zip(got[1:], exact[1:]):
            np.testing.assert_array_equal(g, e)


DIR_CHECKS = [check_directions_against_front, check_bf16_rounding_golden,
              check_operand_rounding, check_storage]


@pytest.mark.parametrize("check", DIR_CHECKS, ids=lambda f: f.__name__)
def test_front_directions_pin(check):
    check(ss2d_front_np)


DIR_MUTATIONS = {
    "direction_1_not_reversed": ("seq = x if k == 0 else x[:, ::-1, :]", "seq = x"),
    "operand_rounding_dropped": (
        'x_dbl = round_storage(u_exact, "bf16") @ round_storage(Wk, "bf16").T',
        "x_dbl = u_exact @ Wk.T"),
    "weight_of_direction_0_used": ("Wk = np.asarray(W_x[k], dtype=np.float64)",
                                   "Wk = np.asarray(W_x[0], dtype=np.float64)"),
    "rounding_ties_away": ("lsb = (u >> 16) & 1", "lsb = np.ones_like(u)"),
}


@pytest.mark.parametrize("name", sorted(DIR_MUTATIONS))
def test_planted_direction_mistake_is_caught(name):
    old, new = DIR_MUTATIONS[name]
    src = inspect.getsource(ss2d_front_np)
    assert src.count(old) == 1, name
    src = src.replace(old, new).replace("from .ss2d_oracle_np import",
                                        "from oracle.ss2d_oracle_np import")
    mod = types.ModuleType(f"front_dir_mutant_{name}")
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    caught = []
    for check in DIR_CHECKS:
        try:
            check(mod)
        except Exception:
            caught.append(check.__name__)
    assert caught, f"planted mistake '{name}' passed every pin"


# ---------------------------------------------------------------------------
# front + scan
# ---------------------------------------------------------------------------
def test_front_scan_one_direction_is_the_composition():
    x, w, b, W_x, w_dt = _problem_k(8, K=1)
    K, D, N = 1, x.shape[2], (W_x.shape[1] - 1) // 2
    rng = np.random.default_rng(9)
    A_log = np.log(np.arange(1, N + 1))[None].repeat(K * D, 0) + rng.uniform(-.5, .5, (K * D, N))
    Dk, bias = rng.uniform(.5, 1.5, K * D), rng.uniform(-4, -2, K * D)
    y = oracle.front_scan(x, w, b, W_x, w_dt, A_log, Dk, bias)
    u, delta, Bs, Cs = ss2d_front_np.front(x, w[0], b[0], W_x[0], w_dt[0])
    want = oracle.selective_scan_fwd(u, delta, A_log, Bs, Cs, Dk, bias, K=1)
    np.testing.assert_allclose(y, want, rtol=1e-13, atol=1e-13)


def test_front_scan_palindrome_reads_both_directions_in_order():
    """A sequence equal to its reverse, and the same weights for both
    directions: direction 1 sees what direction 0 sees, so its output in scan
    order equals direction 0's, and y = y0 + y0 flipped along L."""
    x, w, b, W_x, w_dt = _problem_k(10, K=1)
    x = x + x[:, ::-1, :]
    K, D, N = 2, x.shape[2], (W_x.shape[1] - 1) // 2
    two = [np.concatenate([a, a], axis=0) for a in (w, b, W_x, w_dt)]
    A_log = np.log(np.arange(1, N + 1))[None].repeat(K * D, 0)
    Dk, bias = np.ones(K * D), np.full(K * D, -3.0)
    y = oracle.front_scan(x, *two, A_log, Dk, bias)
    y0 = oracle.front_scan(x, w, b, W_x, w_dt, A_log[:D], Dk[:D], bias[:D])
    np.testing.assert_allclose(y, y0 + y0[:, :, ::-1], rtol=1e-12, atol=1e-12)
    assert np.abs(y0 - y0[:, :, ::-1]).max() > 1e-3   # the flip is visible

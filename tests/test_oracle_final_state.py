"""Pins of the oracle's final states h_L (``oracle.final_states``), the state
after the last step of every direction's scan.

* through the C forward oracle (a separate program): with C = 0 everywhere
  except C = e_n at the last scan step, direction k's output at that step's
  pixel is h_L[n] + Dskip * u;
* L = 1: h = dt * B * u;
* constant inputs: the geometric series dt B u (1 - a^L) / (1 - a)."""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from oracle.ss2d_oracle_np import scan_orders_1d, scan_orders_2d


def _inputs(kind, B, D, H, W, K, N, seed):
    rng = np.random.default_rng(seed)
    L = H * W if kind == "2d" else W
    xshape = (B, D, H, W) if kind == "2d" else (B, D, L)
    return (rng.standard_normal(xshape), rng.standard_normal((B, K, D, L)),
            rng.uniform(-1.0, 1.0, (K * D, N)), rng.standard_normal((B, K, N, L)),
            rng.standard_normal(K * D), rng.uniform(-1.0, 1.0, K * D))


@pytest.mark.parametrize("case", [("2d", 2, 3, 3, 4, 4, 3), ("2d", 1, 2, 2, 5, 2, 2),
                                  ("1d", 2, 3, 1, 7, 2, 4), ("1d", 1, 2, 1, 6, 1, 3)],
                         ids=lambda c: "_".join(map(str, c)))
def test_final_state_through_the_c_forward(case):
    kind, B, D, H, W, K, N = case
    x, delta, A_log, Bs, Dskip, bias = _inputs(kind, B, D, H, W, K, N, seed=11)
    L = H * W if kind == "2d" else W
    hL = oracle.final_states(x, delta, A_log, Bs, bias, K=K, two_d=(kind == "2d"))
    orders = scan_orders_2d(H, W) if kind == "2d" else scan_orders_1d(L)
    fwd = oracle.ss2d_forward if kind == "2d" else oracle.selective_scan_fwd
    u = x.reshape(B, D, L)
    for n in range(N):
        Cs = np.zeros((B, K, N, L))
        Cs[:, :, n, L - 1] = 1.0
        _, yd = fwd(x, delta, A_log, Bs, Cs, Dskip, bias, K=K, return_dirs=True)
        for k in range(K):
            p = orders[k][L - 1]   # pixel of direction k's last step
            got = yd[:, k, :, p] - Dskip[k * D:(k + 1) * D][None] * u[:, :, p]
            np.testing.assert_allclose(hL[:, k, :, n], got, rtol=1e-12, atol=1e-14)


def test_final_state_one_step():
    x, delta, A_log, Bs, _, bias = _inputs("1d", 2, 3, 1, 1, 1, 4, seed=3)
    hL = oracle.final_states(x, delta, A_log, Bs, bias, K=1, two_d=False)
    dt = np.log1p(np.exp(delta[:, 0, :, 0] + bias[None]))
    want = dt[:, :, None] * Bs[:, 0, :, 0][:, None, :] * x[:, :, 0][:, :, None]
    np.testing.assert_allclose(hL[:, 0], want, rtol=1e-13)


def test_final_state_geometric_series():
    L, dz, Al, b, u = 37, 0.3, 0.2, -0.1, 0.8
    x = np.full((1, 1, L), u)
    delta = np.full((1, 1, 1, L), dz)
    Bs = np.full((1, 1, 1, L), 1.5)
    hL = oracle.final_states(x, delta, np.array([[Al]]), Bs, np.array([b]), K=1, two_d=False)
    dt = math.log1p(math.exp(dz + b))
    a = math.exp(-dt * math.exp(Al))
    want = dt * 1.5 * u * (1 - a ** L) / (1 - a)
    assert abs(hL[0, 0, 0, 0] - want) <= 1e-13 * abs(want)


MUTATIONS = {
    "one_step_short": ("        for t in range(L):\n            h = np.exp(",
                       "        for t in range(L - 1):\n            h = np.exp("),
    "scan_order_ignored": ("u = u_pix[:, :, orders[k]]", "u = u_pix"),
    "no_decay": ("h = np.exp(dt[:, :, t, None] * A[None]) * h + \\",
                 "h = h + \\"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_final_state_mistake_is_caught(name):
    import inspect
    import types
    from oracle import ss2d_oracle_np
    old, new = MUTATIONS[name]
    src = inspect.getsource(ss2d_oracle_np.final_states)
    assert src.count(old) == 1, name
    mod = types.ModuleType("fs_mutant")
    mod.__dict__.update(np=np, softplus=ss2d_oracle_np.softplus,
                        scan_orders_1d=scan_orders_1d, scan_orders_2d=scan_orders_2d)
    exec(compile(src.replace(old, new), "<mutant>", "exec"), mod.__dict__)
    real = oracle.final_states
    caught = False
    try:
        oracle.final_states = mod.final_states
        for case in [("2d", 2, 3, 3, 4, 4, 3), ("1d", 2, 3, 1, 7, 2, 4)]:
            try:
                test_final_state_through_the_c_forward(case)
            except AssertionError:
                caught = True
    finally:
        oracle.final_states = real
    assert caught, f"planted mistake '{name}' passed"

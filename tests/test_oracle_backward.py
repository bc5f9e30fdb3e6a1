"""Pins of the float64 backward oracle (``oracle/ss2d_backward_np.py``).

The backward is the gradient of sum(dy * y) for the forward definition; these
checks fix it against things other than itself:

* central finite differences of the C forward oracle (a separate program,
  itself pinned by ``test_oracle_pins.py``) on EVERY input element of small
  2D (K = 4, K = 2, K = 1) and 1D (K = 2, K = 1) problems;
* closed forms of a two-step, one-state scan derived by hand from the
  recurrence;
* planted mistakes in the backward's source, each of which must fail the
  finite-difference check.
"""
from __future__ import annotations

import math
import types

import numpy as np
import pytest

import oracle
from oracle import ss2d_backward_np

NAMES = ("x", "delta", "A_log", "Bs", "Cs", "Dskip", "delta_bias")
GRADS = ("dx", "ddelta", "dA_log", "dBs", "dCs", "dDskip", "ddelta_bias")


def _problem(kind, B, D, H, W, K, N, seed):
    """Inputs with dt of order one (so every term of the gradient matters):
    N(0,1) x, delta, Bs, Cs, dy; A_log ~ U(-1, 1); Dskip ~ N(0,1); bias ~ U(-1, 1)."""
    rng = np.random.default_rng(seed)
    L = H * W if kind == "2d" else W
    xshape = (B, D, H, W) if kind == "2d" else (B, D, L)
    return dict(
        x=rng.standard_normal(xshape),
        delta=rng.standard_normal((B, K, D, L)),
        A_log=rng.uniform(-1.0, 1.0, (K * D, N)),
        Bs=rng.standard_normal((B, K, N, L)),
        Cs=rng.standard_normal((B, K, N, L)),
        Dskip=rng.standard_normal(K * D),
        delta_bias=rng.uniform(-1.0, 1.0, K * D),
    ), rng.standard_normal(xshape)


def _loss(kind, K, inp, dy):
    fn = oracle.ss2d_forward if kind == "2d" else oracle.selective_scan_fwd
    y = fn(*[inp[n] for n in NAMES], K=K)
    return float(np.sum(dy * y))


def _finite_differences(kind, K, inp, dy, eps=1e-6):
    out = {}
    for name, gname in zip(NAMES, GRADS):
        a = inp[name]
        g = np.empty_like(a)
        for i in range(a.size):
            old = a.flat[i]
            a.flat[i] = old + eps
            lp = _loss(kind, K, inp, dy)
            a.flat[i] = old - eps
            lm = _loss(kind, K, inp, dy)
            a.flat[i] = old
            g.flat[i] = (lp - lm) / (2 * eps)
        out[gname] = g
    return out


def _check_against_fd(bwd, kind, K, inp, dy, fd):
    got = bwd(*[inp[n] for n in NAMES], dy, K=K)
    bad = []
    for gname in GRADS:
        a, b = got[gname], fd[gname]
        assert a.shape == b.shape, (gname, a.shape, b.shape)
        # central differences at eps = 1e-6: truncation ~1e-12, rounding ~1e-10
        if not np.all(np.abs(a - b) <= 1e-6 * np.maximum(1.0, np.abs(b))):
            bad.append(gname)
    return bad


FD_CASES = [
    ("2d", 1, 2, 3, 4, 4, 3),   # non-square: the column-major maps differ from their inverses
    ("2d", 2, 1, 2, 3, 2, 2),
    ("2d", 1, 2, 3, 2, 1, 2),
    ("1d", 2, 2, 1, 7, 2, 3),
    ("1d", 1, 3, 1, 5, 1, 4),
]
_FD_CACHE = {}


def _fd_case(case):
    if case not in _FD_CACHE:
        kind, B, D, H, W, K, N = case
        inp, dy = _problem(kind, B, D, H, W, K, N, seed=FD_CASES.index(case))
        _FD_CACHE[case] = (inp, dy, _finite_differences(kind, K, inp, dy))
    return _FD_CACHE[case]


def _bwd_fn(mod, kind):
    return mod.ss2d_backward if kind == "2d" else mod.selective_scan_bwd


@pytest.mark.parametrize("case", FD_CASES, ids=lambda c: "_".join(map(str, c)))
def test_backward_matches_finite_differences(case):
    inp, dy, fd = _fd_case(case)
    bad = _check_against_fd(_bwd_fn(ss2d_backward_np, case[0]), case[0], case[5], inp, dy, fd)
    assert not bad, f"gradients off the finite differences: {bad}"


def test_two_step_closed_form():
    """One channel, one state, L = 2, K = 1, derived by hand:
    s_t = softplus(delta_t + b), A = -e^{A_log}, a_1 = e^{s_1 A};
    h_0 = s_0 B_0 u_0, h_1 = a_1 h_0 + s_1 B_1 u_1, y_t = C_t h_t + D u_t;
    loss = g_0 y_0 + g_1 y_1."""
    u0, u1, d0, d1, b, Al = 0.7, -1.3, 0.4, -0.9, 0.25, 0.3
    B0, B1, C0, C1, Dk, g0, g1 = 1.1, -0.6, 0.8, 1.7, -0.45, 0.9, -1.2

    def sp(z):
        return math.log1p(math.exp(z))

    def sig(z):
        return 1.0 / (1.0 + math.exp(-z))

    s0, s1, A = sp(d0 + b), sp(d1 + b), -math.exp(Al)
    a1 = math.exp(s1 * A)
    h0 = s0 * B0 * u0
    h1 = a1 * h0 + s1 * B1 * u1
    c0 = g0 * C0 + g1 * C1 * a1          # dloss/dh_0
    want = {
        "dx": [g0 * (C0 * s0 * B0 + Dk) + g1 * C1 * a1 * s0 * B0, g1 * (C1 * s1 * B1 + Dk)],
        "ddelta": [c0 * B0 * u0 * sig(d0 + b), g1 * C1 * (A * a1 * h0 + B1 * u1) * sig(d1 + b)],
        "dA_log": [g1 * C1 * h0 * a1 * s1 * A],
        "dBs": [c0 * s0 * u0, g1 * C1 * s1 * u1],
        "dCs": [g0 * h0, g1 * h1],
        "dDskip": [g0 * u0 + g1 * u1],
    }
    want["ddelta_bias"] = [sum(want["ddelta"])]
    got = oracle.selective_scan_bwd(
        np.array([[[u0, u1]]]), np.array([[[[d0, d1]]]]), np.array([[Al]]),
        np.array([[[[B0, B1]]]]), np.array([[[[C0, C1]]]]), np.array([Dk]), np.array([b]),
        np.array([[[g0, g1]]]), K=1)
    for name, w in want.items():
        np.testing.assert_allclose(got[name].reshape(-1), w, rtol=1e-13, atol=1e-15,
                                   err_msg=name)


def test_reverse_direction_is_the_flipped_problem():
    """K = 2 in 1D: direction 1 is direction 0 of the time-reversed sequence
    (with its own parameters), so its gradients are the flipped gradients of
    that K = 1 problem."""
    inp, dy = _problem("1d", 2, 3, 1, 9, 2, 4, seed=7)
    g2 = oracle.selective_scan_bwd(*[inp[n] for n in NAMES], dy, K=2)
    rev = dict(x=inp["x"][:, :, ::-1], delta=inp["delta"][:, 1:2], A_log=inp["A_log"][3:],
               Bs=inp["Bs"][:, 1:2], Cs=inp["Cs"][:, 1:2], Dskip=inp["Dskip"][3:],
               delta_bias=inp["delta_bias"][3:])
    fwd = dict(x=inp["x"], delta=inp["delta"][:, :1], A_log=inp["A_log"][:3],
               Bs=inp["Bs"][:, :1], Cs=inp["Cs"][:, :1], Dskip=inp["Dskip"][:3],
               delta_bias=inp["delta_bias"][:3])
    g_rev = oracle.selective_scan_bwd(*[rev[n] for n in NAMES], dy[:, :, ::-1], K=1)
    g_fwd = oracle.selective_scan_bwd(*[fwd[n] for n in NAMES], dy, K=1)
    np.testing.assert_allclose(g2["dx"], g_fwd["dx"] + g_rev["dx"][:, :, ::-1], rtol=1e-12,
                               atol=1e-14)
    np.testing.assert_allclose(g2["ddelta"][:, 1], g_rev["ddelta"][:, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g2["dBs"][:, 1], g_rev["dBs"][:, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g2["dA_log"][3:], g_rev["dA_log"], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# planted mistakes: each edit of the backward's source must fail the
# finite-difference check on at least one case
# ---------------------------------------------------------------------------
MUTATIONS = {
    "ddt_drops_decay_term": [("(A[None] * a * h_prev + Bt * u[:, :, t, None])",
                              "(Bt * u[:, :, t, None])")],
    "dA_reads_h_t": [("dA += (g * dt[:, :, t, None] * a * h_prev)",
                      "dA += (g * dt[:, :, t, None] * a * hs[:, :, t])")],
    "adjoint_not_decayed": [("        g = g * a\n", "        g = g\n")],
    "skip_term_dropped": [("du[:, :, t] = Dk[None] * gy[:, :, t] + dt", "du[:, :, t] = dt")],
    "softplus_slope_flipped": [("ddelta = ddt * sigmoid(z)", "ddelta = ddt * sigmoid(-z)")],
    "dA_log_chain_dropped": [("dA_log[rows] = dA * A", "dA_log[rows] = dA")],
    "dx_scattered_the_wrong_way": [("dx[:, :, perm] += du", "dx += du[:, :, perm]")],
    "dC_reads_adjoint": [("dC[:, :, t] = (gy[:, :, t, None] * hs[:, :, t])",
                          "dC[:, :, t] = (g * hs[:, :, t])")],
    "dB_without_dt": [("dB[:, :, t] = (g * dt[:, :, t, None] * u[:, :, t, None])",
                       "dB[:, :, t] = (g * u[:, :, t, None])")],
    "dy_not_gathered": [("dy_pix[:, :, perm]", "dy_pix")],
    # the output term joins the adjoint after the decay instead of before it
    "output_term_after_decay": [
        ("        g = g + gy[:, :, t, None] * Ck[:, None, :, t]\n", ""),
        ("        g = g * a\n",
         "        g = g * a\n        g = g + gy[:, :, t, None] * Ck[:, None, :, t]\n")],
    "bias_grad_first_step_only": [("dbias[rows] = dd.sum(axis=(0, 2))",
                                   "dbias[rows] = dd[:, :, 0].sum(axis=0)")],
}


def _mutant(name):
    with open(ss2d_backward_np.__file__) as f:
        src = f.read()
    for old, new in MUTATIONS[name]:
        assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
        src = src.replace(old, new)
    src = src.replace("from .ss2d_oracle_np import", "from oracle.ss2d_oracle_np import")
    mod = types.ModuleType(f"bwd_mutant_{name}")
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_backward_mistake_is_caught(name):
    mod = _mutant(name)
    caught = []
    for case in FD_CASES:
        inp, dy, fd = _fd_case(case)
        try:
            bad = _check_against_fd(_bwd_fn(mod, case[0]), case[0], case[5], inp, dy, fd)
        except Exception as e:   # a mistake that breaks shapes is caught too
            bad = [repr(e)]
        caught += bad
    assert caught, f"planted mistake '{name}' passed every finite-difference check"

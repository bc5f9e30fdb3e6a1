"""Checks that pin the float64 oracle to facts that do not come from the
oracle itself: closed forms, a matrix-exponential discretisation, an O(L^2)
brute force, hand-worked fixtures and exact index-map invariants.

Each check takes an implementation ``impl`` -- a pair of callables with the
oracle's signatures (2D forward, 1D forward) -- and raises AssertionError if
the implementation breaks the pinned fact.  ``tests/test_oracle_pins.py`` runs
them on the C oracle and on its NumPy twin, and on copies of the C oracle with
a planted mistake to show that every plausible mistake is caught.
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# fixtures and small helpers
# --------------------------------------------------------------------------
def read_golden(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, vals = line.partition(":")
            out[key.strip()] = vals.split()
    return out


def array_scan_orders(H: int, W: int) -> list[np.ndarray]:
    """Scan orders built from array reshapes/flips/transposes, following the
    tutorial's CrossScanModule (checked against the hand-written fixture in
    test_scan_orders_fixture)."""
    img = np.arange(H * W).reshape(H, W)
    rm = img.reshape(-1)
    cm = img.transpose(1, 0).reshape(-1)
    return [rm, rm[::-1], cm, cm[::-1]]


def softplus_ref(z: float) -> float:
    """log(1 + e^z) straight from its definition (moderate z only)."""
    return math.log1p(math.exp(z))


def rand_problem(rng, B, D, H, W, K, N, *, one_d=False):
    L = H * W
    x = rng.standard_normal((B, D, L) if one_d else (B, D, H, W))
    delta = rng.standard_normal((B, K, D, L))
    Bs = rng.standard_normal((B, K, N, L))
    Cs = rng.standard_normal((B, K, N, L))
    A_log = rng.uniform(-1.0, 2.5, size=(K * D, N))
    Dskip = rng.standard_normal(K * D)
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=K * D))
    delta_bias = np.log(np.expm1(dt))
    return dict(x=x, delta=delta, A_log=A_log, Bs=Bs, Cs=Cs, Dskip=Dskip,
                delta_bias=delta_bias)


def call2d(impl, p, K, **kw):
    return impl[0](p["x"], p["delta"], p["A_log"], p["Bs"], p["Cs"],
                   p["Dskip"], p["delta_bias"], K=K, **kw)


def call1d(impl, p, K, **kw):
    return impl[1](p["x"], p["delta"], p["A_log"], p["Bs"], p["Cs"],
                   p["Dskip"], p["delta_bias"], K=K, **kw)


def expm_taylor(M: np.ndarray) -> np.ndarray:
    """Matrix exponential by scaling and squaring with a Taylor series,
    float64, no library routine: exp(M) = (exp(M / 2^s))^(2^s)."""
    norm = np.abs(M).sum(axis=1).max()
    s = max(0, int(math.ceil(math.log2(norm))) + 1) if norm > 0 else 0
    A = M / (2.0 ** s)
    E = np.eye(M.shape[0])
    term = np.eye(M.shape[0])
    for j in range(1, 30):
        term = term @ A / j
        E = E + term
    for _ in range(s):
        E = E @ E
    return E


# --------------------------------------------------------------------------
# the pins
# --------------------------------------------------------------------------
def pin_hand_worked(impl):
    """Two-step scan worked by hand (tests/golden/hand_worked_1d.txt)."""
    g = read_golden("hand_worked_1d.txt")
    u = np.array([float(v) for v in g["u"]]).reshape(1, 1, 2)
    a = np.array([float(v) for v in g["a"]])
    b = np.array([float(v) for v in g["b"]])
    p = dict(x=u, delta=np.zeros((1, 1, 1, 2)), A_log=np.zeros((1, 1)),
             Bs=np.ones((1, 1, 1, 2)), Cs=np.ones((1, 1, 1, 2)),
             Dskip=np.ones(1), delta_bias=np.zeros(1))
    y = call1d(impl, p, K=1).reshape(-1)
    want = a * math.log(2.0) + b
    np.testing.assert_allclose(y, want, rtol=1e-15, atol=0)


def pin_integrator_scan_orders(impl, H=3, W=5):
    """With A = 0 (A_log = -inf), N = 1, B = C = 1 and dt = 1 the scan is a
    running sum, so direction k's output at pixel p is the sum of the inputs
    met along that direction's order up to p.  Pins all four orders, their
    inverses and the direction indexing of delta/Bs/Cs/params."""
    rng = np.random.default_rng(11)
    B, D, K, N, L = 2, 3, 4, 1, H * W
    x = rng.integers(-9, 10, size=(B, D, H, W)).astype(np.float64)
    one = math.log(math.expm1(1.0))             # softplus^-1(1)
    p = dict(x=x, delta=np.zeros((B, K, D, L)),
             A_log=np.full((K * D, N), -np.inf), Bs=np.ones((B, K, N, L)),
             Cs=np.ones((B, K, N, L)), Dskip=np.zeros(K * D),
             delta_bias=np.full(K * D, one))
    y, yd = call2d(impl, p, K=4, return_dirs=True)
    seq = x.reshape(B, D, L)
    rows = seq
    cols = x.transpose(0, 1, 3, 2).reshape(B, D, L)
    want = [np.cumsum(rows, -1).reshape(B, D, H, W),
            np.cumsum(rows[..., ::-1], -1)[..., ::-1].reshape(B, D, H, W),
            np.cumsum(cols, -1).reshape(B, D, W, H).transpose(0, 1, 3, 2),
            np.cumsum(cols[..., ::-1], -1)[..., ::-1]
            .reshape(B, D, W, H).transpose(0, 1, 3, 2)]
    for k in range(4):
        np.testing.assert_allclose(yd[:, k].reshape(B, D, H, W), want[k],
                                   rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, ((want[0] + want[1]) + want[2]) + want[3],
                               rtol=1e-12, atol=1e-12)
    # 1D: forward running sum and reversed running sum
    u = seq[:, :, :7].copy()
    p1 = dict(p, x=u, delta=np.zeros((B, 2, D, 7)), Bs=np.ones((B, 2, 1, 7)),
              Cs=np.ones((B, 2, 1, 7)), A_log=np.full((2 * D, 1), -np.inf),
              Dskip=np.zeros(2 * D), delta_bias=np.full(2 * D, one))
    y1, yd1 = call1d(impl, p1, K=2, return_dirs=True)
    np.testing.assert_allclose(yd1[:, 0], np.cumsum(u, -1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(yd1[:, 1], np.cumsum(u[..., ::-1], -1)[..., ::-1],
                               rtol=1e-12, atol=1e-12)


def pin_single_step_closed_form(impl):
    """L = 1 (H = W = 1): every direction sees the one pixel once, so
    y = sum_k [ sum_n C_kn * dt_k * B_kn * u + D_k * u ], dt_k = softplus."""
    rng = np.random.default_rng(12)
    B, D, K, N = 3, 4, 4, 5
    p = rand_problem(rng, B, D, 1, 1, K, N)
    y = call2d(impl, p, K=4)
    want = np.zeros((B, D))
    for b in range(B):
        for d in range(D):
            u = p["x"][b, d, 0, 0]
            tot = 0.0
            for k in range(K):
                kd = k * D + d
                dt = softplus_ref(p["delta"][b, k, d, 0] + p["delta_bias"][kd])
                s = sum(p["Cs"][b, k, n, 0] * dt * p["Bs"][b, k, n, 0] * u
                        for n in range(N))
                tot += s + p["Dskip"][kd] * u
            want[b, d] = tot
    np.testing.assert_allclose(y.reshape(B, D), want, rtol=1e-13, atol=1e-14)


def pin_geometric_series(impl):
    """Constant dt, B, C and u along a sequence: with a = exp(dt*A_n),
    h_n(t) = dt B_n u (1 - a^t)/(1 - a) after t steps, so
    y(t) = sum_n C_n h_n(t) + D u.  Checked on the 1D forward and reversed
    directions (the reversed one reaches pixel p after L - p steps)."""
    rng = np.random.default_rng(13)
    B, D, K, N, L = 2, 3, 2, 4, 40
    u = np.repeat(rng.standard_normal((B, D, 1)), L, axis=2)
    delta = np.repeat(rng.standard_normal((B, K, D, 1)), L, axis=3)
    Bc = rng.standard_normal((B, K, N, 1))
    Cc = rng.standard_normal((B, K, N, 1))
    A_log = rng.uniform(-2.0, 2.0, size=(K * D, N))
    Dskip = rng.standard_normal(K * D)
    delta_bias = rng.uniform(-3.0, 1.0, size=K * D)
    p = dict(x=u, delta=delta, A_log=A_log, Bs=np.repeat(Bc, L, 3),
             Cs=np.repeat(Cc, L, 3), Dskip=Dskip, delta_bias=delta_bias)
    y, yd = call1d(impl, p, K=2, return_dirs=True)
    want = np.zeros((B, K, D, L))
    for b in range(B):
        for k in range(K):
            for d in range(D):
                kd = k * D + d
                dt = softplus_ref(delta[b, k, d, 0] + delta_bias[kd])
                uu = u[b, d, 0]
                for pix in range(L):
                    t = pix + 1 if k == 0 else L - pix
                    acc = 0.0
                    for n in range(N):
                        A = -math.exp(A_log[kd, n])
                        # (1 - a^t)/(1 - a) = expm1(t dt A)/expm1(dt A)
                        g = math.expm1(t * dt * A) / math.expm1(dt * A)
                        acc += Cc[b, k, n, 0] * dt * Bc[b, k, n, 0] * uu * g
                    want[b, k, d, pix] = acc + Dskip[kd] * uu
    np.testing.assert_allclose(yd, want, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(y, want[:, 0] + want[:, 1], rtol=1e-11, atol=1e-12)


def pin_matrix_exponential_discretisation(impl):
    """Zero-order hold from the continuous system ("Vision Mamba ..." summary,
    section 4.1): exp([[dt A, dt B], [0, 0]]) has top-left block exp(dt A) and
    top-right block (dt A)^-1 (exp(dt A) - I) dt B.  A recurrence driven by
    those blocks (computed here by a Taylor matrix exponential) must equal
    the implementation in both discretisation modes: 'zoh' uses both blocks,
    'euler' (the path) uses the top-left block with dt*B."""
    rng = np.random.default_rng(14)
    B, D, K, N, L = 1, 2, 1, 3, 6
    p = rand_problem(rng, B, D, 1, L, K, N, one_d=True)
    p["delta_bias"] = rng.uniform(-2.0, 1.0, size=K * D)   # larger dt
    for mode in ("euler", "zoh"):
        y = call1d(impl, p, K=1, bbar=mode)
        want = np.zeros((B, D, L))
        for d in range(D):
            A = -np.exp(p["A_log"][d])
            h = np.zeros(N)
            for t in range(L):
                dt = softplus_ref(p["delta"][0, 0, d, t] + p["delta_bias"][d])
                Bt = p["Bs"][0, 0, :, t]
                M = np.zeros((N + 1, N + 1))
                M[:N, :N] = np.diag(dt * A)
                M[:N, N] = dt * Bt
                E = expm_taylor(M)
                assert np.abs(E[:N, :N] - np.diag(np.diag(E[:N, :N]))).max() < 1e-15
                Abar = np.diag(E[:N, :N])
                Bbar = E[:N, N] if mode == "zoh" else dt * Bt
                u = p["x"][0, d, t]
                h = Abar * h + Bbar * u
                want[0, d, t] = p["Cs"][0, 0, :, t] @ h + p["Dskip"][d] * u
        np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-13)


def pin_convolution_form(impl):
    """Time-varying generalisation of the global-convolution form ("Vision
    Mamba ..." summary, section 4.1): unrolling the recurrence gives
    y_t = sum_{s<=t} sum_n C_{t,n} (prod_{r=s+1..t} a_{r,n}) dt_s B_{s,n} u_s
    + D u_t, a_{r,n} = exp(dt_r A_n).  Brute force, O(L^2 N), on the 1D
    forward and reversed directions and on all four 2D directions."""
    rng = np.random.default_rng(15)

    def conv(u, dt, A, Bk, Ck, Dk):
        L = u.shape[0]
        a = np.exp(dt[:, None] * A[None, :])            # (L, N)
        y = np.zeros(L)
        for t in range(L):
            tot = Dk * u[t]
            for s in range(t + 1):
                prod = np.prod(a[s + 1:t + 1], axis=0)  # empty -> ones
                tot += np.sum(Ck[:, t] * prod * dt[s] * Bk[:, s] * u[s])
            y[t] = tot
        return y

    # 1D, K = 2
    B, D, K, N, L = 1, 2, 2, 3, 9
    p = rand_problem(rng, B, D, 1, L, K, N, one_d=True)
    y, yd = call1d(impl, p, K=2, return_dirs=True)
    for k in range(K):
        for d in range(D):
            kd = k * D + d
            u = p["x"][0, d] if k == 0 else p["x"][0, d, ::-1]
            dt = np.array([softplus_ref(v + p["delta_bias"][kd])
                           for v in p["delta"][0, k, d]])
            ys = conv(u, dt, -np.exp(p["A_log"][kd]), p["Bs"][0, k], p["Cs"][0, k],
                      p["Dskip"][kd])
            got = yd[0, k, d] if k == 0 else yd[0, k, d, ::-1]
            np.testing.assert_allclose(got, ys, rtol=1e-12, atol=1e-13)
    # 2D, K = 4, non-square
    H, W = 2, 3
    B, D, K, N = 1, 2, 4, 2
    p = rand_problem(rng, B, D, H, W, K, N)
    y, yd = call2d(impl, p, K=4, return_dirs=True)
    orders = array_scan_orders(H, W)
    for k in range(4):
        for d in range(D):
            kd = k * D + d
            u = p["x"][0, d].reshape(-1)[orders[k]]
            dt = np.array([softplus_ref(v + p["delta_bias"][kd])
                           for v in p["delta"][0, k, d]])
            ys = conv(u, dt, -np.exp(p["A_log"][kd]), p["Bs"][0, k], p["Cs"][0, k],
                      p["Dskip"][kd])
            np.testing.assert_allclose(yd[0, k, d][orders[k]], ys, rtol=1e-12,
                                       atol=1e-13)
    np.testing.assert_allclose(y.reshape(B, D, -1), yd.sum(1), rtol=1e-13, atol=1e-13)


def pin_identity_scan(impl):
    """With Bs = 0 the states stay 0 and only the skip term remains; with
    Dskip = 1, cross_merge(cross_scan(x)) = 4x (2x for the 1D K = 2 case),
    bit-exact for integer-valued inputs."""
    rng = np.random.default_rng(16)
    for (H, W) in [(3, 5), (4, 4), (1, 7)]:
        B, D, K, N, L = 2, 3, 4, 3, H * W
        p = rand_problem(rng, B, D, H, W, K, N)
        p["x"] = rng.integers(-50, 51, size=(B, D, H, W)).astype(np.float64)
        p["Bs"] = np.zeros((B, K, N, L))
        p["Dskip"] = np.ones(K * D)
        y = call2d(impl, p, K=4)
        assert np.array_equal(y, 4.0 * p["x"]), "2D identity scan is not 4x"
    B, D, K, N, L = 2, 3, 2, 2, 11
    p = rand_problem(rng, B, D, 1, L, K, N, one_d=True)
    p["x"] = rng.integers(-50, 51, size=(B, D, L)).astype(np.float64)
    p["Cs"] = np.zeros((B, K, N, L))
    p["Dskip"] = np.ones(K * D)
    y = call1d(impl, p, K=2)
    assert np.array_equal(y, 2.0 * p["x"]), "1D identity scan is not 2x"


def pin_reversal_invariant(impl):
    """Rotating the map by 180 degrees reverses both the row-major and the
    column-major order.  So direction 1 on rot180(x) sees exactly the sequence
    direction 0 sees on x (same delta/B/C/params), and its pixel-order output
    is rot180 of direction 0's; likewise direction 3 vs direction 2.
    Bit-exact: the same arithmetic runs in the same order."""
    rng = np.random.default_rng(17)
    H, W = 3, 4
    B, D, K, N = 2, 2, 4, 3
    p = rand_problem(rng, B, D, H, W, K, N)
    q = {k: v.copy() for k, v in p.items()}
    q["x"] = p["x"][:, :, ::-1, ::-1].copy()
    for (src, dst) in [(0, 1), (2, 3)]:
        q["delta"][:, dst] = p["delta"][:, src]
        q["Bs"][:, dst] = p["Bs"][:, src]
        q["Cs"][:, dst] = p["Cs"][:, src]
        for name in ("A_log", "Dskip", "delta_bias"):
            q[name][dst * D:(dst + 1) * D] = p[name][src * D:(src + 1) * D]
    _, yp = call2d(impl, p, K=4, return_dirs=True)
    _, yq = call2d(impl, q, K=4, return_dirs=True)
    for (src, dst) in [(0, 1), (2, 3)]:
        a = yp[:, src].reshape(B, D, H, W)[:, :, ::-1, ::-1]
        b = yq[:, dst].reshape(B, D, H, W)
        assert np.array_equal(a, b), f"direction {dst} is not the 180-degree image of {src}"
    # 1D: direction 1 on flip(u) equals flip of direction 0 on u
    L = 8
    p = rand_problem(rng, 1, 2, 1, L, 2, 3, one_d=True)
    q = {k: v.copy() for k, v in p.items()}
    q["x"] = p["x"][:, :, ::-1].copy()
    q["delta"][:, 1] = p["delta"][:, 0]
    q["Bs"][:, 1] = p["Bs"][:, 0]
    q["Cs"][:, 1] = p["Cs"][:, 0]
    for name in ("A_log", "Dskip", "delta_bias"):
        q[name][2:4] = p[name][0:2]
    _, yp = call1d(impl, p, K=2, return_dirs=True)
    _, yq = call1d(impl, q, K=2, return_dirs=True)
    assert np.array_equal(yp[:, 0][..., ::-1], yq[:, 1])


def pin_linearity(impl):
    """delta, B and C do not depend on x, so y is linear in x: doubling x
    doubles y exactly (power-of-two scaling), and y(x1 + x2) = y(x1) + y(x2)."""
    rng = np.random.default_rng(18)
    p = rand_problem(rng, 2, 3, 3, 4, 4, 4)
    y1 = call2d(impl, p, K=4)
    y2 = call2d(impl, dict(p, x=2.0 * p["x"]), K=4)
    assert np.array_equal(y2, 2.0 * y1)
    x2 = rng.standard_normal(p["x"].shape)
    ys = call2d(impl, dict(p, x=p["x"] + x2), K=4)
    yb = call2d(impl, dict(p, x=x2), K=4)
    np.testing.assert_allclose(ys, y1 + yb, rtol=1e-12, atol=1e-12)


def pin_decomposition(impl):
    """SS2D with K = 4 equals four 1D single-direction scans run on explicitly
    cross-scanned copies, mapped back and added in the order k = 0..3."""
    rng = np.random.default_rng(19)
    H, W = 3, 5
    B, D, K, N = 2, 2, 4, 3
    p = rand_problem(rng, B, D, H, W, K, N)
    y = call2d(impl, p, K=4)
    orders = array_scan_orders(H, W)
    total = None
    for k in range(4):
        rows = slice(k * D, (k + 1) * D)
        u = p["x"].reshape(B, D, -1)[:, :, orders[k]]
        q = dict(x=u, delta=p["delta"][:, k:k + 1], Bs=p["Bs"][:, k:k + 1],
                 Cs=p["Cs"][:, k:k + 1], A_log=p["A_log"][rows],
                 Dskip=p["Dskip"][rows], delta_bias=p["delta_bias"][rows])
        ys = call1d(impl, q, K=1)
        yk = np.empty_like(ys)
        yk[:, :, orders[k]] = ys
        total = yk if total is None else total + yk
    np.testing.assert_allclose(y.reshape(B, D, -1), total, rtol=1e-14, atol=1e-14)


def pin_extreme_softplus(impl):
    """softplus must neither overflow for large arguments nor lose small
    ones: dt = softplus(800) is 800, dt = softplus(-40) is e^-40.  A single
    step (L = 1, N = 1, B = C = 1, Dskip = 0) returns y = dt * u."""
    for z, dt in [(800.0, 800.0), (-40.0, math.exp(-40.0)), (0.0, math.log(2.0))]:
        p = dict(x=np.ones((1, 1, 1)), delta=np.full((1, 1, 1, 1), z),
                 A_log=np.zeros((1, 1)), Bs=np.ones((1, 1, 1, 1)),
                 Cs=np.ones((1, 1, 1, 1)), Dskip=np.zeros(1),
                 delta_bias=np.zeros(1))
        y = call1d(impl, p, K=1)
        np.testing.assert_allclose(y.reshape(-1), [dt], rtol=1e-14, atol=0)


def pin_gate(impl):
    """The gate multiplies the merged output by SiLU(z) = z * sigmoid(z)
    pointwise.  With the identity scan (Bs = 0, Dskip = 1) the ungated output
    is 4x (2x for the 1D K = 2 case), so the gated output is a closed form:
    sigmoid(ln 3) = 3/4 gives SiLU(ln 3) = (3/4) ln 3 and SiLU(-ln 3) =
    -(1/4) ln 3; SiLU(0) = 0; SiLU(40) is 40 to 1e-15 relative; SiLU(-40)
    is -40 e^-40 to 1e-15 relative (no overflow, the small value kept).
    Without z the output is the ungated one."""
    rng = np.random.default_rng(20)
    ln3 = math.log(3.0)
    table = {ln3: 0.75 * ln3, -ln3: -0.25 * ln3, 0.0: 0.0, 40.0: 40.0,
             -40.0: -40.0 * math.exp(-40.0)}
    keys = np.array(sorted(table))
    H, W, B, D, K, N = 3, 4, 2, 3, 4, 2
    p = rand_problem(rng, B, D, H, W, K, N)
    p["x"] = rng.integers(-8, 9, size=(B, D, H, W)).astype(np.float64)
    p["Bs"] = np.zeros((B, K, N, H * W))
    p["Dskip"] = np.ones(K * D)
    z = keys[rng.integers(0, len(keys), size=p["x"].shape)]
    want = 4.0 * p["x"] * np.vectorize(table.get)(z)
    y = call2d(impl, p, K=4, z=z)
    np.testing.assert_allclose(y, want, rtol=1e-15, atol=0)
    assert np.array_equal(call2d(impl, p, K=4), 4.0 * p["x"]), "ungated output changed"
    # 1D, K = 2
    L = 10
    p = rand_problem(rng, B, D, 1, L, 2, N, one_d=True)
    p["x"] = rng.integers(-8, 9, size=(B, D, L)).astype(np.float64)
    p["Cs"] = np.zeros((B, 2, N, L))
    p["Dskip"] = np.ones(2 * D)
    z = keys[rng.integers(0, len(keys), size=p["x"].shape)]
    y = call1d(impl, p, K=2, z=z)
    np.testing.assert_allclose(y, 2.0 * p["x"] * np.vectorize(table.get)(z), rtol=1e-15, atol=0)


ALL_PINS = [pin_hand_worked, pin_integrator_scan_orders, pin_single_step_closed_form,
            pin_geometric_series, pin_matrix_exponential_discretisation,
            pin_convolution_form, pin_identity_scan, pin_reversal_invariant,
            pin_linearity, pin_decomposition, pin_extreme_softplus, pin_gate]

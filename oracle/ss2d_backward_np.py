"""NumPy float64 backward (reverse-mode gradient) of the SS2D forward path --
TEST INFRASTRUCTURE ONLY.

The pages ask for a backward pass that recomputes the scan instead of storing
the states in HBM ("Vision Mamba ..." summary, section 4.4, Memory and IO
Efficiency).  They give no gradient formulas; the gradient is fixed by the
forward definition alone (see ``ss2d_oracle.c``):

    dt_t = softplus(delta_t + bias)                      (per direction k, channel d)
    h_t  = exp(dt_t * A) * h_{t-1} + dt_t * B_t * u_t    (A = -exp(A_log), h_{-1} = 0)
    y_t  = C_t . h_t + Dskip * u_t,   u_t = x[pixel_k(t)],  y = sum_k y_k[scan_k^-1]

This module is that definition differentiated by the chain rule, step by
step, in the plainest form: the forward sweep keeps every state h_t (float64),
the reverse sweep walks t = L-1 .. 0 carrying g = dLoss/dh_t, with the loss
sum(dy * y) for a given cotangent dy.  At step t:

    g      += dy_t * C_t                          (y_t reads h_t)
    dC_t   += dy_t * h_t                          (summed over the channels d)
    dB_t   += g * dt_t * u_t                      (summed over d)
    du_t    = Dskip * dy_t + dt_t * sum_n g_n B_t,n
    ddt_t   = sum_n g_n * (A_n * exp(dt_t A_n) * h_{t-1},n + B_t,n * u_t)
    dA_n   += g_n * dt_t * exp(dt_t A_n) * h_{t-1},n
    dDskip += dy_t * u_t
    g      *= exp(dt_t * A)                       (h_t reads h_{t-1})

then ddelta_t = ddt_t * sigmoid(delta_t + bias) (softplus' = sigmoid),
dbias = sum_t ddelta_t, dA_log = dA * A (dA/dA_log = A), and dx gathers du_k
of every direction back to its pixel (the adjoint of the cross_scan gather).
The parameter gradients are summed over the batch.

Pinned in ``tests/test_oracle_backward.py`` against central finite differences
of the C forward oracle (a separate program) on every input element of small
problems, and against closed forms of one- and two-step scans derived by hand.
"""
from __future__ import annotations

import numpy as np

from .ss2d_oracle_np import scan_orders_1d, scan_orders_2d, softplus


def sigmoid(z):
    """1 / (1 + e^-z), written with e^-|z| so that it never overflows."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def _direction_backward(u, gy, dt, z, A, Bk, Ck, Dk):
    """One direction in scan order.  u, gy, dt, z: (B, D, L); A: (D, N);
    Bk, Ck: (B, N, L); Dk: (D,).  Returns du, ddelta (B, D, L), dA (D, N),
    dB, dC (B, N, L), dDk (D,)."""
    Bb, D, L = u.shape
    N = A.shape[1]
    # forward sweep, every state kept
    hs = np.empty((Bb, D, L, N))
    h = np.zeros((Bb, D, N))
    for t in range(L):
        a = np.exp(dt[:, :, t, None] * A[None])
        h = a * h + dt[:, :, t, None] * Bk[:, None, :, t] * u[:, :, t, None]
        hs[:, :, t] = h
    # reverse sweep
    du = np.empty((Bb, D, L))
    ddt = np.empty((Bb, D, L))
    dA = np.zeros((D, N))
    dB = np.empty((Bb, N, L))
    dC = np.empty((Bb, N, L))
    dDk = np.zeros(D)
    g = np.zeros((Bb, D, N))
    for t in range(L - 1, -1, -1):
        a = np.exp(dt[:, :, t, None] * A[None])
        h_prev = hs[:, :, t - 1] if t > 0 else np.zeros((Bb, D, N))
        Bt = Bk[:, None, :, t]
        g = g + gy[:, :, t, None] * Ck[:, None, :, t]
        dC[:, :, t] = (gy[:, :, t, None] * hs[:, :, t]).sum(axis=1)
        dB[:, :, t] = (g * dt[:, :, t, None] * u[:, :, t, None]).sum(axis=1)
        du[:, :, t] = Dk[None] * gy[:, :, t] + dt[:, :, t] * (g * Bt).sum(-1)
        ddt[:, :, t] = (g * (A[None] * a * h_prev + Bt * u[:, :, t, None])).sum(-1)
        dA += (g * dt[:, :, t, None] * a * h_prev).sum(axis=0)
        dDk += (gy[:, :, t] * u[:, :, t]).sum(axis=0)
        g = g * a
    ddelta = ddt * sigmoid(z)
    return du, ddelta, dA, dB, dC, dDk


def _backward(u_pix, orders, delta, A_log, Bs, Cs, Dskip, delta_bias, dy_pix, K):
    Bb, D, L = u_pix.shape
    N = A_log.shape[1]
    dx = np.zeros((Bb, D, L))
    ddelta = np.empty((Bb, K, D, L))
    dA_log = np.empty((K * D, N))
    dBs = np.empty((Bb, K, N, L))
    dCs = np.empty((Bb, K, N, L))
    dDskip = np.empty(K * D)
    dbias = np.empty(K * D)
    for k in range(K):
        perm = orders[k]
        rows = slice(k * D, (k + 1) * D)
        A = -np.exp(A_log[rows])
        z = delta[:, k] + delta_bias[rows][None, :, None]
        du, dd, dA, dB, dC, dDk = _direction_backward(
            u_pix[:, :, perm], dy_pix[:, :, perm], softplus(z), z, A, Bs[:, k], Cs[:, k],
            Dskip[rows])
        dx[:, :, perm] += du
        ddelta[:, k] = dd
        dA_log[rows] = dA * A
        dBs[:, k] = dB
        dCs[:, k] = dC
        dDskip[rows] = dDk
        dbias[rows] = dd.sum(axis=(0, 2))
    return dict(dx=dx, ddelta=ddelta, dA_log=dA_log, dBs=dBs, dCs=dCs, dDskip=dDskip,
                ddelta_bias=dbias)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def ss2d_backward(x, delta, A_log, Bs, Cs, Dskip, delta_bias, dy, *, K=4):
    """Gradients of sum(dy * ss2d_forward(...)) with respect to every input.
    x, dy: (B, D, H, W).  Returns a dict of float64 arrays shaped like the
    inputs: dx, ddelta, dA_log, dBs, dCs, dDskip, ddelta_bias."""
    x = _f64(x)
    Bb, D, H, W = x.shape
    g = _backward(x.reshape(Bb, D, H * W), scan_orders_2d(H, W)[:K], _f64(delta), _f64(A_log),
                  _f64(Bs), _f64(Cs), _f64(Dskip), _f64(delta_bias),
                  _f64(dy).reshape(Bb, D, H * W), K)
    g["dx"] = g["dx"].reshape(Bb, D, H, W)
    return g


def selective_scan_bwd(u, delta, A_log, Bs, Cs, Dskip, delta_bias, dy, *, K=2):
    """The same for the 1D scan (K = 1: forward; K = 2: forward + reversed).
    u, dy: (B, D, L)."""
    u = _f64(u)
    return _backward(u, scan_orders_1d(u.shape[2])[:K], _f64(delta), _f64(A_log), _f64(Bs),
                     _f64(Cs), _f64(Dskip), _f64(delta_bias), _f64(dy), K)

"""NumPy float64 write-up of the SS2D forward path -- TEST INFRASTRUCTURE ONLY.

A second, independent statement of the same definition as ``ss2d_oracle.c``
(see that file's header for the page passages each step follows).  Here the
four scan orders are built the way the pages build them -- reshape, flip and
transpose of the H x W map ("VMamba架构解析", section 1, cross_scan; "Vision
Mamba" tutorial, CrossScanModule) -- instead of by index arithmetic, and the
recurrence runs over the scan index with all channels of a direction as one
array ("Vision Mamba" tutorial, SelectiveSSM._selective_scan).
"""
from __future__ import annotations

import numpy as np


def softplus(z):
    """log(1 + e^z), written so that e^z never overflows."""
    z = np.asarray(z, dtype=np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def silu(z):
    """z * sigmoid(z), written with the logistic function of |z| so that e^x
    never overflows (the Vim block's gate; see ss2d_oracle.c)."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    sig = np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return z * sig


def scan_orders_2d(H: int, W: int) -> list[np.ndarray]:
    """Pixel index visited at each scan step for the four SS2D directions,
    in the stacking order [row-major, its flip, column-major, its flip]."""
    pix = np.arange(H * W).reshape(H, W)
    row_major = pix.reshape(-1)
    col_major = pix.T.reshape(-1)
    return [row_major, row_major[::-1].copy(), col_major, col_major[::-1].copy()]


def scan_orders_1d(L: int) -> list[np.ndarray]:
    seq = np.arange(L)
    return [seq, seq[::-1].copy()]


def _scan_direction(u_scan, dt, A, Bk, Ck, Dk, bbar):
    """u_scan, dt: (B, D, L) in scan order; A: (D, N); Bk, Ck: (B, N, L);
    Dk: (D,).  Returns y in scan order, (B, D, L)."""
    Bb, D, L = u_scan.shape
    N = A.shape[1]
    h = np.zeros((Bb, D, N))
    y = np.empty((Bb, D, L))
    for t in range(L):
        dA = np.exp(dt[:, :, t, None] * A[None, :, :])
        if bbar == "euler":
            dB = dt[:, :, t, None] * Bk[:, None, :, t]
        else:
            safeA = np.where(A == 0.0, 1.0, A)
            zoh = np.expm1(dt[:, :, t, None] * A[None]) / safeA[None]
            zoh = np.where(A[None] == 0.0, dt[:, :, t, None], zoh)
            dB = zoh * Bk[:, None, :, t]
        h = dA * h + dB * u_scan[:, :, t, None]
        y[:, :, t] = (h * Ck[:, None, :, t]).sum(-1) + Dk[None, :] * u_scan[:, :, t]
    return y


def _forward(u_pix, orders, delta, A_log, Bs, Cs, Dskip, delta_bias, K, bbar):
    Bb, D, L = u_pix.shape
    y = np.zeros((Bb, D, L))
    ydirs = np.empty((Bb, K, D, L))
    for k in range(K):
        perm = orders[k]
        rows = slice(k * D, (k + 1) * D)
        A = -np.exp(A_log[rows])
        dt = softplus(delta[:, k] + delta_bias[rows][None, :, None])
        yk_scan = _scan_direction(u_pix[:, :, perm], dt, A, Bs[:, k], Cs[:, k],
                                  Dskip[rows], bbar)
        yk_pix = np.empty_like(yk_scan)
        yk_pix[:, :, perm] = yk_scan
        ydirs[:, k] = yk_pix
        y = y + yk_pix
    return y, ydirs


def ss2d_forward(x, delta, A_log, Bs, Cs, Dskip, delta_bias, K=4,
                 bbar="euler", return_dirs=False, z=None):
    x = np.asarray(x, dtype=np.float64)
    Bb, D, H, W = x.shape
    y, yd = _forward(x.reshape(Bb, D, H * W), scan_orders_2d(H, W),
                     np.asarray(delta, np.float64), np.asarray(A_log, np.float64),
                     np.asarray(Bs, np.float64), np.asarray(Cs, np.float64),
                     np.asarray(Dskip, np.float64),
                     np.asarray(delta_bias, np.float64), K, bbar)
    y = y.reshape(Bb, D, H, W)
    if z is not None:
        y = y * silu(z)
    return (y, yd) if return_dirs else y


def selective_scan_fwd(u, delta, A_log, Bs, Cs, Dskip, delta_bias, K=2,
                       bbar="euler", return_dirs=False, z=None):
    u = np.asarray(u, dtype=np.float64)
    Bb, D, L = u.shape
    y, yd = _forward(u, scan_orders_1d(L), np.asarray(delta, np.float64),
                     np.asarray(A_log, np.float64), np.asarray(Bs, np.float64),
                     np.asarray(Cs, np.float64), np.asarray(Dskip, np.float64),
                     np.asarray(delta_bias, np.float64), K, bbar)
    if z is not None:
        y = y * silu(z)
    return (y, yd) if return_dirs else y


def final_states(x, delta, A_log, Bs, delta_bias, *, K, two_d=True):
    """The state after the last step of every direction's scan, h_L
    (B, K, D, N), float64: the recurrence of the forward (dt = softplus(delta
    + bias), h = exp(dt A) h + dt B u from h = 0) run to the end of direction
    k's scan order (the state a continued scan would start from)."""
    x = np.asarray(x, dtype=np.float64)
    Bb, D = x.shape[:2]
    if two_d:
        H, W = x.shape[2:]
        L, orders = H * W, scan_orders_2d(H, W)
    else:
        L = x.shape[2]
        orders = scan_orders_1d(L)
    u_pix = x.reshape(Bb, D, L)
    delta = np.asarray(delta, np.float64)
    A_log = np.asarray(A_log, np.float64)
    Bs = np.asarray(Bs, np.float64)
    delta_bias = np.asarray(delta_bias, np.float64)
    N = A_log.shape[1]
    out = np.zeros((Bb, K, D, N))
    for k in range(K):
        rows = slice(k * D, (k + 1) * D)
        A = -np.exp(A_log[rows])
        dt = softplus(delta[:, k] + delta_bias[rows][None, :, None])
        u = u_pix[:, :, orders[k]]
        h = np.zeros((Bb, D, N))
        for t in range(L):
            h = np.exp(dt[:, :, t, None] * A[None]) * h + \
                dt[:, :, t, None] * Bs[:, k][:, None, :, t] * u[:, :, t, None]
        out[:, k] = h
    return out

"""NumPy float64 write-up of the front that feeds the selective scan in the
tutorial's SelectiveSSM -- TEST INFRASTRUCTURE ONLY.

"Vision Mamba" tutorial, section "Background: State Space Models and Mamba",
SelectiveSSM.forward: from the input branch x (B, L, D) of in_proj,

  1. a causal depthwise conv1d of width d_conv (4), with bias: the layer pads
     d_conv - 1 zeros on both sides and keeps the first L outputs, so output
     step l sees inputs l - d_conv + 1 .. l (zeros before the sequence start):
         c[b, l, d] = bias[d] + sum_j w[d, j] * x[b, l - (d_conv - 1) + j, d]
     (a cross-correlation, as a convolution layer computes it);
  2. SiLU: u = c * sigmoid(c);
  3. x_proj: a Linear from D to 1 + 2N without bias, split into
     (dt_raw (1), B (N), C (N));
  4. dt_proj: a Linear from 1 to D with bias; softplus of it is the step.

In the scan's terms (the inputs of ``selective_scan_fwd`` with K = 1):
u (B, D, L) = SiLU(conv(x)) transposed, delta[b, 0, d, l] = w_dt[d] *
dt_raw[b, l] (the bias of dt_proj is the scan's delta_bias), Bs, Cs
(B, 1, N, L).  The matrix products are NumPy's; everything else is written
out step by step.

Pinned in ``tests/test_oracle_front.py``: the conv against NumPy's own
``convolve`` per channel, its impulse response and causality, x_proj against
selector weights and linearity, and planted mistakes.
"""
from __future__ import annotations

import numpy as np

from .ss2d_oracle_np import silu


def causal_depthwise_conv(x, w, bias):
    """x (B, L, D), w (D, d_conv), bias (D,) -> (B, L, D)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    Bb, L, D = x.shape
    kc = w.shape[1]
    out = np.empty((Bb, L, D))
    for l in range(L):
        acc = np.array(bias, dtype=np.float64)[None, :].repeat(Bb, axis=0)
        for j in range(kc):
            src = l - (kc - 1) + j
            if src >= 0:
                acc = acc + w[None, :, j] * x[:, src, :]
        out[:, l, :] = acc
    return out


def front(x, conv_w, conv_b, W_x, w_dt):
    """x (B, L, D) input branch; conv_w (D, d_conv), conv_b (D,); W_x
    (1 + 2N, D) the x_proj weight; w_dt (D,) the dt_proj weight.  Returns the
    scan's inputs in its layout: u (B, D, L), delta (B, 1, D, L), Bs and Cs
    (B, 1, N, L), all float64."""
    W_x = np.asarray(W_x, dtype=np.float64)
    N = (W_x.shape[0] - 1) // 2
    u_bld = silu(causal_depthwise_conv(x, conv_w, conv_b))          # (B, L, D)
    x_dbl = u_bld @ W_x.T                                           # (B, L, 1 + 2N)
    dt_raw = x_dbl[:, :, 0]                                         # (B, L)
    Bm = x_dbl[:, :, 1:1 + N]
    Cm = x_dbl[:, :, 1 + N:1 + 2 * N]
    delta = np.asarray(w_dt, dtype=np.float64)[None, :, None] * dt_raw[:, None, :]
    return (np.ascontiguousarray(u_bld.transpose(0, 2, 1)),
            np.ascontiguousarray(delta[:, None]),
            np.ascontiguousarray(Bm.transpose(0, 2, 1)[:, None]),
            np.ascontiguousarray(Cm.transpose(0, 2, 1)[:, None]))

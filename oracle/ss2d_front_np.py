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

``front_directions`` is the bidirectional form of the Vim block ("Vision
Mamba ..." summary, section 4.3): each of the K directions runs its own conv1d
and projections on its own sequence, the input itself (k = 0) or the input
reversed along L (k = 1), and the results come out in that direction's scan
order.  It states two readings the pages leave open, about precision:

* ``operand="bf16"``: x_proj multiplies bfloat16 operands -- u and W_x each
  rounded to bfloat16 (nearest, ties to even) from their exact values -- and
  sums the products exactly (the tensor-core form of the product, with a
  float32 accumulator on the GPU); ``operand="f64"`` keeps them exact;
* ``storage``: u, which the scan reads, is stored in the input's dtype
  ("f32", "bf16" or "f16", rounded to nearest even from the exact value), or
  kept exact (None).
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


def round_storage(a, storage):
    """a (float64) rounded to a storage dtype, returned as float64 values:
    "f32" and "f16" by NumPy's casts (nearest, ties to even), "bf16" by
    keeping the upper 16 bits of the float32 value after rounding to nearest
    with ties to even; None returns a unchanged."""
    a = np.asarray(a, dtype=np.float64)
    if storage is None:
        return a
    if storage == "f32":
        return a.astype(np.float32).astype(np.float64)
    if storage == "f16":
        return a.astype(np.float16).astype(np.float64)
    if storage == "bf16":
        u = np.ascontiguousarray(a.astype(np.float32)).view(np.uint32).astype(np.uint64)
        lsb = (u >> 16) & 1
        r = (((u + 0x7FFF + lsb) >> 16) << 16).astype(np.uint32)
        return r.view(np.float32).astype(np.float64)
    raise ValueError(f"unknown storage {storage!r}")


def front_directions(x, conv_w, conv_b, W_x, w_dt, *, storage=None, operand="f64"):
    """x (B, L, D) input branch; conv_w (K, D, d_conv), conv_b (K, D), W_x
    (K, 1 + 2N, D), w_dt (K, D): direction k's conv, x_proj and dt_proj
    weights.  Direction 0 reads the sequence as it is, direction 1 reversed.
    Returns, in each direction's scan order: u (B, K, D, L) as stored (see
    ``storage``), delta (B, K, D, L) = w_dt[k, d] * dt_raw[b, k, l], Bs and Cs
    (B, K, N, L), all float64."""
    x = np.asarray(x, dtype=np.float64)
    conv_w = np.asarray(conv_w, dtype=np.float64)
    K = conv_w.shape[0]
    outs = []
    for k in range(K):
        seq = x if k == 0 else x[:, ::-1, :]
        u_exact = silu(causal_depthwise_conv(seq, conv_w[k], conv_b[k]))   # (B, L, D)
        Wk = np.asarray(W_x[k], dtype=np.float64)
        if operand == "bf16":
            x_dbl = round_storage(u_exact, "bf16") @ round_storage(Wk, "bf16").T
        elif operand == "f64":
            x_dbl = u_exact @ Wk.T
        else:
            raise ValueError(f"unknown operand {operand!r}")
        N = (Wk.shape[0] - 1) // 2
        dt_raw = x_dbl[:, :, 0]                                      # (B, L)
        delta = np.asarray(w_dt[k], dtype=np.float64)[None, :, None] * dt_raw[:, None, :]
        outs.append((round_storage(u_exact, storage).transpose(0, 2, 1), delta,
                     x_dbl[:, :, 1:1 + N].transpose(0, 2, 1),
                     x_dbl[:, :, 1 + N:1 + 2 * N].transpose(0, 2, 1)))
    return tuple(np.ascontiguousarray(np.stack([o[i] for o in outs], axis=1))
                 for i in range(4))

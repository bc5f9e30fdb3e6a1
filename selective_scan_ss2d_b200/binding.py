"""Thin ctypes binding of the C ABI in include/ss2d.h.

Argument marshalling only: every step of the forward pass runs in the CUDA
library.  Tensors are torch tensors, either all on the current CUDA device
(asynchronous on the current stream) or all in host memory (the library
copies in, computes on the current device, copies out and synchronises).
There is no CPU fallback: if the library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch


SS2D_F32 = 0
SS2D_BF16 = 1
NOALLOC_SCRATCH_BYTES = 96 * 1024 * 1024   # SS2D_NOALLOC_SCRATCH_BYTES of the C header
SS2D_F16 = 2
_DTYPES = {torch.float32: SS2D_F32, torch.bfloat16: SS2D_BF16, torch.float16: SS2D_F16}

_lock = threading.Lock()
_lib = None


class SS2DError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"ss2d status {status}: {message}")
        self.status = status


_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib",
                         "libss2d_b200.so")


def lib_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _LIB_PATH
            if not os.path.exists(path):
                raise RuntimeError(
                    f"CUDA library {path} is missing: build it with "
                    "`python -m selective_scan_ss2d_b200.build`")
            L = ctypes.CDLL(path)
            vp, fp, i = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
            fwd = [vp, vp, fp, vp, vp, fp, fp, fp]
            L.ss2d_forward.argtypes = fwd + [i] * 7 + [vp]
            L.ss2d_forward.restype = i
            L.ss2d_forward_ex.argtypes = fwd + [i] * 7 + [vp, i]
            L.ss2d_forward_ex.restype = i
            L.selective_scan_fwd.argtypes = fwd + [i] * 6 + [vp]
            L.selective_scan_fwd.restype = i
            L.selective_scan_fwd_ex.argtypes = fwd + [i] * 6 + [vp, i]
            L.selective_scan_fwd_ex.restype = i
            L.ss2d_scan_directions.argtypes = fwd + [i] * 8 + [vp, i]
            gfwd = fwd[:7] + [vp] + fwd[7:]   # the gate z before y
            L.ss2d_forward_gated.argtypes = gfwd + [i] * 7 + [vp]
            L.ss2d_forward_gated.restype = i
            L.selective_scan_fwd_gated.argtypes = gfwd + [i] * 6 + [vp]
            L.selective_scan_fwd_gated.restype = i
            L.ss2d_scan_directions.restype = i
            L.ss2d_forward_final_state.argtypes = fwd + [fp] + [i] * 7 + [vp, i]
            L.ss2d_forward_final_state.restype = i
            L.selective_scan_fwd_final_state.argtypes = fwd + [fp] + [i] * 6 + [vp, i]
            L.selective_scan_fwd_final_state.restype = i
            bwd = fwd[:7] + [fp] + [fp] * 7   # dy, then the seven gradients
            L.ss2d_backward.argtypes = bwd + [i] * 7 + [vp]
            L.ss2d_backward.restype = i
            L.selective_scan_bwd.argtypes = bwd + [i] * 6 + [vp]
            L.selective_scan_bwd.restype = i
            L.ss2d_plan.argtypes = [i] * 8 + [ctypes.POINTER(ctypes.c_int)] * 3
            L.ss2d_plan.restype = i
            L.ss2d_forward_noalloc.argtypes = fwd + [i] * 7 + [vp]
            L.ss2d_forward_noalloc.restype = i
            L.ss2d_forward_timed.argtypes = fwd + [i] * 8 + [vp, i, ctypes.POINTER(ctypes.c_float)]
            L.ss2d_forward_timed.restype = i
            L.ss2d_num_variants.argtypes = []
            L.ss2d_num_variants.restype = i
            L.ss2d_variant_name.argtypes = [i]
            L.ss2d_variant_name.restype = ctypes.c_char_p
            L.ss2d_pick_variant.argtypes = [i] * 7
            L.ss2d_pick_variant.restype = i
            L.selective_scan_fwd_front.argtypes = [vp] + [fp] * 8 + [i] * 6 + [vp]
            L.selective_scan_fwd_front.restype = i
            L.selective_scan_fwd_front_timed.argtypes = ([vp] + [fp] * 8 + [i] * 6 +
                                                         [vp, ctypes.POINTER(ctypes.c_float)])
            L.selective_scan_fwd_front_timed.restype = i
            L.ss2d_front_project.argtypes = [vp, fp, fp, fp, vp, fp, fp, fp] + [i] * 6 + [vp]
            L.ss2d_front_project.restype = i
            L.ss2d_check_waits.argtypes = []
            L.ss2d_check_waits.restype = i
            L.ss2d_wait_selftest.argtypes = [i, vp]
            L.ss2d_wait_selftest.restype = i
            L.ss2d_status_string.argtypes = [i]
            L.ss2d_status_string.restype = ctypes.c_char_p
            L.ss2d_last_error.argtypes = []
            L.ss2d_last_error.restype = ctypes.c_char_p
            _lib = L
        return _lib


def ss2d_status_string(status: int) -> str:
    return lib().ss2d_status_string(int(status)).decode()


def ss2d_num_variants() -> int:
    return lib().ss2d_num_variants()


def ss2d_variant_name(i: int) -> str:
    return lib().ss2d_variant_name(int(i)).decode()


def ss2d_pick_variant(two_d: bool, B: int, D: int, H: int, W: int, N: int, K: int) -> int:
    return lib().ss2d_pick_variant(int(bool(two_d)), B, D, H, W, N, K)


def _check(status: int):
    if status != 0:
        L = lib()
        msg = L.ss2d_status_string(status).decode()
        detail = L.ss2d_last_error().decode()
        raise SS2DError(status, msg + (f" -- {detail}" if detail and status in (-7, -8, -11) else ""))


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr()) if t.numel() > 0 else ctypes.c_void_p(0)


def _prepare(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y, xdims):
    streamed = (x, delta, Bs, Cs)
    dt = x.dtype
    if dt not in _DTYPES:
        raise TypeError(f"x must be float32, bfloat16 or float16, got {dt}")
    for t in streamed:
        if t.dtype != dt:
            raise TypeError("x, delta, Bs and Cs must share one dtype")
    for t in (A_log, Dskip, delta_bias):
        if t.dtype != torch.float32:
            raise TypeError("A_log, Dskip and delta_bias must be float32")
    tensors = list(streamed) + [A_log, Dskip, delta_bias]
    on_gpu = x.is_cuda
    for t in tensors:
        if t.is_cuda != on_gpu or (on_gpu and t.device != x.device):
            raise ValueError("all tensors must be on the same device (or all on the host)")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
    if y is None:
        y = torch.empty(xdims, dtype=torch.float32, device=x.device,
                        pin_memory=(not on_gpu and x.is_pinned()))
    if y.dtype != torch.float32 or tuple(y.shape) != tuple(xdims) or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous float32 tensor of shape {tuple(xdims)}")
    if y.is_cuda != on_gpu:
        raise ValueError("y must live where the inputs live")
    return y, _DTYPES[dt], on_gpu


def _stream(on_gpu, device, stream):
    if stream is not None:
        return ctypes.c_void_p(stream if isinstance(stream, int) else stream.cuda_stream)
    if on_gpu:
        return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    return ctypes.c_void_p(0)


def ss2d_forward(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y=None, *, stream=None,
                 variant: int = -1):
    """SS2D forward (cross_scan -> selective scan -> cross_merge).

    x (B,D,H,W); delta (B,K,D,L) and Bs, Cs (B,K,N,L) in each direction's
    scan order; A_log (K*D,N), Dskip and delta_bias (K*D,) float32.
    Returns y (B,D,H,W) float32."""
    B, D, H, W = x.shape
    K, N = delta.shape[1], Bs.shape[2]
    L = H * W
    if tuple(delta.shape) != (B, K, D, L) or tuple(Bs.shape) != (B, K, N, L) \
            or tuple(Cs.shape) != (B, K, N, L) or tuple(A_log.shape) != (K * D, N) \
            or tuple(Dskip.shape) != (K * D,) or tuple(delta_bias.shape) != (K * D,):
        raise ValueError("inconsistent shapes for ss2d_forward")
    y, dt, on_gpu = _prepare(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y, (B, D, H, W))
    st = _stream(on_gpu, x.device, stream)
    rc = lib().ss2d_forward_ex(_ptr(x), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs),
                               _ptr(Dskip), _ptr(delta_bias), _ptr(y), B, D, H, W, N, K,
                               dt, st, int(variant))
    _check(rc)
    return y


def ss2d_forward_noalloc(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y, *, stream=None):
    """ss2d_forward without any allocation by the library: scratch lives in a
    fixed device buffer of NOALLOC_SCRATCH_BYTES per device (SS2DError with
    status -11 when the problem needs more).  Device tensors only, y given by
    the caller; calls on one device must not overlap in time."""
    B, D, H, W = x.shape
    K, N = delta.shape[1], Bs.shape[2]
    L = H * W
    if tuple(delta.shape) != (B, K, D, L) or tuple(Bs.shape) != (B, K, N, L) \
            or tuple(Cs.shape) != (B, K, N, L) or tuple(A_log.shape) != (K * D, N) \
            or tuple(Dskip.shape) != (K * D,) or tuple(delta_bias.shape) != (K * D,):
        raise ValueError("inconsistent shapes for ss2d_forward_noalloc")
    if y is None:
        raise ValueError("ss2d_forward_noalloc needs a caller-provided y")
    y, dt, on_gpu = _prepare(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y, (B, D, H, W))
    st = _stream(on_gpu, x.device, stream)
    rc = lib().ss2d_forward_noalloc(_ptr(x), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs),
                                    _ptr(Dskip), _ptr(delta_bias), _ptr(y), B, D, H, W, N, K,
                                    dt, st)
    _check(rc)
    return y


def selective_scan_fwd(u, delta, A_log, Bs, Cs, Dskip, delta_bias, y=None, *, stream=None,
                       variant: int = -1):
    """1D selective scan, K = 1 (forward) or 2 (forward + reversed, added).

    u (B,D,L); delta (B,K,D,L); Bs, Cs (B,K,N,L) in each direction's scan
    order.  Returns y (B,D,L) float32."""
    B, D, L = u.shape
    K, N = delta.shape[1], Bs.shape[2]
    if tuple(delta.shape) != (B, K, D, L) or tuple(Bs.shape) != (B, K, N, L) \
            or tuple(Cs.shape) != (B, K, N, L) or tuple(A_log.shape) != (K * D, N) \
            or tuple(Dskip.shape) != (K * D,) or tuple(delta_bias.shape) != (K * D,):
        raise ValueError("inconsistent shapes for selective_scan_fwd")
    y, dt, on_gpu = _prepare(u, delta, A_log, Bs, Cs, Dskip, delta_bias, y, (B, D, L))
    st = _stream(on_gpu, u.device, stream)
    rc = lib().selective_scan_fwd_ex(_ptr(u), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs),
                                     _ptr(Dskip), _ptr(delta_bias), _ptr(y), B, D, L, N, K,
                                     dt, st, int(variant))
    _check(rc)
    return y


def _check_gate(z, x):
    if z.dtype != x.dtype or tuple(z.shape) != tuple(x.shape) or not z.is_contiguous() \
            or z.device != x.device:
        raise ValueError("z must be a contiguous tensor of x's dtype, shape and device")


def ss2d_forward_gated(x, delta, A_log, Bs, Cs, Dskip, delta_bias, z, y=None, *, stream=None):
    """ss2d_forward, then y * SiLU(z) (z in x's layout and dtype).  Device
    tensors only."""
    B, D, H, W = x.shape
    K, N = delta.shape[1], Bs.shape[2]
    L = H * W
    if tuple(delta.shape) != (B, K, D, L) or tuple(Bs.shape) != (B, K, N, L) \
            or tuple(Cs.shape) != (B, K, N, L) or tuple(A_log.shape) != (K * D, N) \
            or tuple(Dskip.shape) != (K * D,) or tuple(delta_bias.shape) != (K * D,):
        raise ValueError("inconsistent shapes for ss2d_forward_gated")
    _check_gate(z, x)
    y, dt, on_gpu = _prepare(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y, (B, D, H, W))
    st = _stream(on_gpu, x.device, stream)
    rc = lib().ss2d_forward_gated(_ptr(x), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs),
                                  _ptr(Dskip), _ptr(delta_bias), _ptr(z), _ptr(y), B, D, H, W,
                                  N, K, dt, st)
    _check(rc)
    return y


def selective_scan_fwd_gated(u, delta, A_log, Bs, Cs, Dskip, delta_bias, z, y=None, *,
                             stream=None):
    """selective_scan_fwd, then y * SiLU(z) (z in u's layout and dtype).
    Device tensors only."""
    B, D, L = u.shape
    K, N = delta.shape[1], Bs.shape[2]
    if tuple(delta.shape) != (B, K, D, L) or tuple(Bs.shape) != (B, K, N, L) \
            or tuple(Cs.shape) != (B, K, N, L) or tuple(A_log.shape) != (K * D, N) \
            or tuple(Dskip.shape) != (K * D,) or tuple(delta_bias.shape) != (K * D,):
        raise ValueError("inconsistent shapes for selective_scan_fwd_gated")
    _check_gate(z, u)
    y, dt, on_gpu = _prepare(u, delta, A_log, Bs, Cs, Dskip, delta_bias, y, (B, D, L))
    st = _stream(on_gpu, u.device, stream)
    rc = lib().selective_scan_fwd_gated(_ptr(u), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs),
                                        _ptr(Dskip), _ptr(delta_bias), _ptr(z), _ptr(y), B, D,
                                        L, N, K, dt, st)
    _check(rc)
    return y


def ss2d_scan_directions(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y_dir=None, *,
                         two_d: bool = True, stream=None, variant: int = -1):
    """cross_scan + selective scan without the merge: each direction's output
    in pixel order, (B,K,D,H,W) (2D) or (B,K,D,L) (1D).  CUDA tensors only."""
    if two_d:
        B, D, H, W = x.shape
    else:
        B, D, L1 = x.shape
        H, W = 1, L1
    K, N = delta.shape[1], Bs.shape[2]
    L = H * W
    if tuple(delta.shape) != (B, K, D, L) or tuple(Bs.shape) != (B, K, N, L) \
            or tuple(Cs.shape) != (B, K, N, L) or tuple(A_log.shape) != (K * D, N) \
            or tuple(Dskip.shape) != (K * D,) or tuple(delta_bias.shape) != (K * D,):
        raise ValueError("inconsistent shapes for ss2d_scan_directions")
    odims = (B, K, D, H, W) if two_d else (B, K, D, L)
    y_dir, dt, on_gpu = _prepare(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y_dir, odims)
    st = _stream(on_gpu, x.device, stream)
    rc = lib().ss2d_scan_directions(_ptr(x), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs),
                                    _ptr(Dskip), _ptr(delta_bias), _ptr(y_dir), B, D, H, W,
                                    N, K, dt, int(bool(two_d)), st, int(variant))
    _check(rc)
    return y_dir


def ss2d_plan(two_d: bool, B: int, D: int, H: int, W: int, N: int, K: int,
              variant: int = -1) -> dict:
    """Execution plan of a call: steps per chunk, chunks, kernel launches."""
    lc, nc, nl = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().ss2d_plan(int(bool(two_d)), B, D, H, W, N, K, int(variant), ctypes.byref(lc),
                           ctypes.byref(nc), ctypes.byref(nl)))
    return {"chunk_len": lc.value, "num_chunks": nc.value, "launches": nl.value}


def ss2d_forward_timed(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y, *, two_d: bool = True,
                       stream=None, variant: int = -1) -> list:
    """One forward call on CUDA tensors with per-launch device times in ms:
    [chunk state pass, carry, scan pass, cross_merge] (-1 = not launched).
    Blocking (measurement helper)."""
    if two_d:
        B, D, H, W = x.shape
    else:
        B, D, W = x.shape
        H = 1
    K, N = delta.shape[1], Bs.shape[2]
    y, dt, on_gpu = _prepare(x, delta, A_log, Bs, Cs, Dskip, delta_bias, y, tuple(x.shape))
    st = _stream(on_gpu, x.device, stream)
    ms = (ctypes.c_float * 4)()
    _check(lib().ss2d_forward_timed(_ptr(x), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs),
                                    _ptr(Dskip), _ptr(delta_bias), _ptr(y), B, D, H, W, N, K,
                                    dt, int(bool(two_d)), st, int(variant), ms))
    return [float(v) for v in ms]


GRAD_NAMES = ("dx", "ddelta", "dA_log", "dBs", "dCs", "dDskip", "ddelta_bias")


def _backward(fn, name, x, delta, A_log, Bs, Cs, Dskip, delta_bias, dy, dims, stream):
    K, N = delta.shape[1], Bs.shape[2]
    B, D = x.shape[0], x.shape[1]
    L = 1
    for v in x.shape[2:]:
        L *= v
    if tuple(delta.shape) != (B, K, D, L) or tuple(Bs.shape) != (B, K, N, L) \
            or tuple(Cs.shape) != (B, K, N, L) or tuple(A_log.shape) != (K * D, N) \
            or tuple(Dskip.shape) != (K * D,) or tuple(delta_bias.shape) != (K * D,):
        raise ValueError(f"inconsistent shapes for {name}")
    if dy.dtype != torch.float32 or tuple(dy.shape) != tuple(x.shape) or not dy.is_contiguous() \
            or dy.device != x.device:
        raise ValueError("dy must be a contiguous float32 tensor of x's shape and device")
    _, dt, on_gpu = _prepare(x, delta, A_log, Bs, Cs, Dskip, delta_bias, dy, tuple(x.shape))
    if not on_gpu:
        raise ValueError(f"{name} takes device tensors only")
    f32 = dict(dtype=torch.float32, device=x.device)
    g = dict(dx=torch.empty(tuple(x.shape), **f32), ddelta=torch.empty(tuple(delta.shape), **f32),
             dA_log=torch.empty((K * D, N), **f32), dBs=torch.empty(tuple(Bs.shape), **f32),
             dCs=torch.empty(tuple(Cs.shape), **f32), dDskip=torch.empty((K * D,), **f32),
             ddelta_bias=torch.empty((K * D,), **f32))
    st = _stream(True, x.device, stream)
    rc = fn(_ptr(x), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs), _ptr(Dskip),
            _ptr(delta_bias), _ptr(dy), *[_ptr(g[n]) for n in GRAD_NAMES], B, D, *dims, N, K,
            dt, st)
    _check(rc)
    return g


def ss2d_backward(x, delta, A_log, Bs, Cs, Dskip, delta_bias, dy, *, stream=None):
    """Gradients of sum(dy * ss2d_forward(...)) with respect to every input.
    Device tensors only; dy float32 of x's shape.  Returns a dict of float32
    tensors: dx, ddelta, dA_log, dBs, dCs, dDskip, ddelta_bias."""
    H, W = x.shape[2], x.shape[3]
    return _backward(lib().ss2d_backward, "ss2d_backward", x, delta, A_log, Bs, Cs, Dskip,
                     delta_bias, dy, (H, W), stream)


def selective_scan_bwd(u, delta, A_log, Bs, Cs, Dskip, delta_bias, dy, *, stream=None):
    """Gradients of sum(dy * selective_scan_fwd(...)); the dict's "dx" is the
    gradient with respect to u."""
    return _backward(lib().selective_scan_bwd, "selective_scan_bwd", u, delta, A_log, Bs, Cs,
                     Dskip, delta_bias, dy, (u.shape[2],), stream)


def forward_final_state(x, delta, A_log, Bs, Cs, Dskip, delta_bias, *, stream=None,
                        variant: int = -1):
    """ss2d_forward (x 4-D) or selective_scan_fwd (x 3-D) that also returns
    the final states: (y, h_last), h_last (B,K,D,N) float32 the state after
    the last step of every direction's scan.  Device tensors only."""
    two_d = x.dim() == 4
    B, D = x.shape[0], x.shape[1]
    K, N = delta.shape[1], Bs.shape[2]
    L = x.shape[2] * x.shape[3] if two_d else x.shape[2]
    if tuple(delta.shape) != (B, K, D, L) or tuple(Bs.shape) != (B, K, N, L) \
            or tuple(Cs.shape) != (B, K, N, L) or tuple(A_log.shape) != (K * D, N) \
            or tuple(Dskip.shape) != (K * D,) or tuple(delta_bias.shape) != (K * D,):
        raise ValueError("inconsistent shapes for forward_final_state")
    y, dt, on_gpu = _prepare(x, delta, A_log, Bs, Cs, Dskip, delta_bias, None, tuple(x.shape))
    if not on_gpu:
        raise ValueError("forward_final_state takes device tensors only")
    h_last = torch.empty((B, K, D, N), dtype=torch.float32, device=x.device)
    st = _stream(True, x.device, stream)
    args = [_ptr(x), _ptr(delta), _ptr(A_log), _ptr(Bs), _ptr(Cs), _ptr(Dskip), _ptr(delta_bias),
            _ptr(y), _ptr(h_last)]
    if two_d:
        rc = lib().ss2d_forward_final_state(*args, B, D, x.shape[2], x.shape[3], N, K, dt, st,
                                            int(variant))
    else:
        rc = lib().selective_scan_fwd_final_state(*args, B, D, L, N, K, dt, st, int(variant))
    _check(rc)
    return y, h_last


def _front_checks(x, conv_w, conv_b, W_x, w_dt, K, what):
    if x.dtype not in _DTYPES:
        raise TypeError(f"x must be float32, bfloat16 or float16, got {x.dtype}")
    B, L, D = x.shape
    R = W_x.shape[1] if W_x.dim() == 3 else -1
    N = (R - 1) // 2
    if tuple(conv_w.shape) != (K, D, 4) or tuple(conv_b.shape) != (K, D) \
            or W_x.dim() != 3 or tuple(W_x.shape) != (K, 1 + 2 * N, D) or N < 1 \
            or (w_dt is not None and tuple(w_dt.shape) != (K, D)):
        raise ValueError(f"inconsistent shapes for {what}")
    for t in (conv_w, conv_b, W_x) + ((w_dt,) if w_dt is not None else ()):
        if t.dtype != torch.float32:
            raise TypeError("conv_w, conv_b, W_x and w_dt must be float32")
    for t in (x, conv_w, conv_b, W_x) + ((w_dt,) if w_dt is not None else ()):
        if not t.is_cuda or t.device != x.device:
            raise ValueError(f"{what} takes device tensors on one device")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
    return B, L, D, N


def selective_scan_fwd_front(x, conv_w, conv_b, W_x, w_dt, A_log, Dskip, delta_bias, y=None,
                             *, stream=None):
    """The fused front (causal depthwise conv1d + SiLU + x_proj on the tensor
    cores + dt_proj) of every direction, then its selective scan, directions
    summed.  x (B, L, D) input branch; conv_w (K, D, 4), conv_b (K, D), W_x
    (K, 1 + 2N, D), w_dt (K, D); A_log (K*D, N), Dskip, delta_bias (K*D,)
    float32.  Returns y (B, D, L) float32.  Device tensors only."""
    K = conv_w.shape[0]
    B, L, D, N = _front_checks(x, conv_w, conv_b, W_x, w_dt, K, "selective_scan_fwd_front")
    for t in (A_log, Dskip, delta_bias):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("A_log, Dskip and delta_bias must be contiguous float32 device tensors")
    if tuple(A_log.shape) != (K * D, N) or tuple(Dskip.shape) != (K * D,) \
            or tuple(delta_bias.shape) != (K * D,):
        raise ValueError("inconsistent shapes for selective_scan_fwd_front")
    if y is None:
        y = torch.empty((B, D, L), dtype=torch.float32, device=x.device)
    if y.dtype != torch.float32 or tuple(y.shape) != (B, D, L) or not y.is_contiguous() \
            or not y.is_cuda:
        raise ValueError(f"y must be a contiguous float32 device tensor of shape {(B, D, L)}")
    st = _stream(True, x.device, stream)
    rc = lib().selective_scan_fwd_front(_ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(W_x),
                                        _ptr(w_dt), _ptr(A_log), _ptr(Dskip), _ptr(delta_bias),
                                        _ptr(y), B, D, L, N, K, _DTYPES[x.dtype], st)
    _check(rc)
    return y


def selective_scan_fwd_front_timed(x, conv_w, conv_b, W_x, w_dt, A_log, Dskip, delta_bias, y,
                                   *, stream=None):
    """selective_scan_fwd_front into y, synchronised; returns the device
    milliseconds of [front kernel, scan passes, cross_merge] (-1: not run)."""
    K = conv_w.shape[0]
    B, L, D, N = _front_checks(x, conv_w, conv_b, W_x, w_dt, K, "selective_scan_fwd_front")
    if y.dtype != torch.float32 or tuple(y.shape) != (B, D, L) or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous float32 device tensor of shape {(B, D, L)}")
    ms = (ctypes.c_float * 3)()
    st = _stream(True, x.device, stream)
    rc = lib().selective_scan_fwd_front_timed(_ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(W_x),
                                              _ptr(w_dt), _ptr(A_log), _ptr(Dskip),
                                              _ptr(delta_bias), _ptr(y), B, D, L, N, K,
                                              _DTYPES[x.dtype], st, ms)
    _check(rc)
    return [ms[0], ms[1], ms[2]]


def ss2d_front_project(x, conv_w, conv_b, W_x, *, stream=None):
    """The front alone: returns (u (B, K, D, L) in x's dtype, dt_raw (B, K, L),
    Bs, Cs (B, K, N, L) float32), each in its direction's scan order.  L must
    be a multiple of 8.  Device tensors only."""
    K = conv_w.shape[0]
    B, L, D, N = _front_checks(x, conv_w, conv_b, W_x, None, K, "ss2d_front_project")
    dev = x.device
    u = torch.empty((B, K, D, L), dtype=x.dtype, device=dev)
    dt_raw = torch.empty((B, K, L), dtype=torch.float32, device=dev)
    Bs = torch.empty((B, K, N, L), dtype=torch.float32, device=dev)
    Cs = torch.empty((B, K, N, L), dtype=torch.float32, device=dev)
    st = _stream(True, dev, stream)
    rc = lib().ss2d_front_project(_ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(W_x), _ptr(u),
                                  _ptr(dt_raw), _ptr(Bs), _ptr(Cs), B, D, L, N, K,
                                  _DTYPES[x.dtype], st)
    _check(rc)
    return u, dt_raw, Bs, Cs


def ss2d_check_waits() -> int:
    """Status of the library's bounded waits on the current device since the
    last check (0, or -8 if one ran out); clears the record."""
    return lib().ss2d_check_waits()


def ss2d_wait_selftest(limit_us: int, *, stream=None) -> None:
    """Enqueue the wait that cannot complete, limited to limit_us."""
    _check(lib().ss2d_wait_selftest(int(limit_us), _stream(True, None, stream)))

"""Float64 CPU oracle for the SS2D forward path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library in
``selective_scan_ss2d_b200``) never imports, links or calls it; the two share
no code.  Only the seeded input generator (``selective_scan_ss2d_b200.workloads``,
which holds none of the method's arithmetic) feeds both.

Two independent write-ups of the same definition live here:

* ``ss2d_oracle.c`` -- sequential C, float64, the timed baseline; index maps
  by integer arithmetic.  Loaded through ctypes (:func:`ss2d_forward`,
  :func:`selective_scan_fwd`).
* ``ss2d_oracle_np.py`` -- NumPy, float64, sequential over the scan index;
  index maps built from array reshapes, transposes and flips.

What they compute and which page passage each step follows is stated in the
header of ``ss2d_oracle.c``.  ``ss2d_backward_np.py`` (:func:`ss2d_backward`,
:func:`selective_scan_bwd`) is the float64 reverse-mode gradient of the same
forward definition, pinned against finite differences of the C forward;
:func:`final_states` gives the state after each direction's last step.
``ss2d_front_np.py`` writes out the front that feeds the scan in the
tutorial's SelectiveSSM (causal depthwise conv1d, SiLU, x_proj, dt_proj) and
its per-direction form of the Vim block; :func:`front_scan` runs it and then
the scan of every direction, pinned in ``tests/test_oracle_front.py``.  Every part is pinned by ``tests/test_oracle_pins.py``
against closed forms, a matrix-exponential discretisation, an O(L^2) brute
force and exact index-map invariants; parity is pinned for every function
(no function here is "parity unpinned").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .ss2d_backward_np import selective_scan_bwd, ss2d_backward  # noqa: F401
from .ss2d_front_np import front_directions  # noqa: F401
from .ss2d_oracle_np import final_states  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ss2d_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libss2d_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``ss2d_oracle.c`` into ``oracle/_build/libss2d_oracle.so``.

    Plain IEEE float64 (-O2, no fast-math); OpenMP only splits independent
    (b, d) channels across host threads.
    """
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-shared", "-fPIC", "-std=c11", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def compile_variant(src_text: str, out_path: str) -> ctypes.CDLL:
    """Compile an edited copy of the oracle source (used only by the test that
    plants mistakes in the oracle to show the pins catch them)."""
    src_path = out_path + ".c"
    with open(src_path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off",
                    "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", out_path,
                    src_path, "-lm"], check=True)
    return _bind(ctypes.CDLL(out_path))


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


_dp = ctypes.POINTER(ctypes.c_double)


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    i = ctypes.c_int
    lib.oracle_ss2d_forward.argtypes = [_dp] * 7 + [_dp, _dp] + [i] * 8
    lib.oracle_ss2d_forward.restype = i
    lib.oracle_selective_scan_fwd.argtypes = [_dp] * 7 + [_dp, _dp] + [i] * 7
    lib.oracle_selective_scan_fwd.restype = i
    lib.oracle_softplus.argtypes = [ctypes.c_double]
    lib.oracle_softplus.restype = ctypes.c_double
    lib.oracle_scan_pixel.argtypes = [i, i, ctypes.c_int64, i, i]
    lib.oracle_scan_pixel.restype = ctypes.c_int64
    lib.oracle_silu.argtypes = [ctypes.c_double]
    lib.oracle_silu.restype = ctypes.c_double
    lib.oracle_gate.argtypes = [_dp, _dp, ctypes.c_int64]
    lib.oracle_gate.restype = i
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = i
    return lib


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


_BBAR = {"euler": 0, "zoh": 1}


def _gate(y: np.ndarray, z, lb) -> np.ndarray:
    z = _f64(z)
    assert z.shape == y.shape
    st = lb.oracle_gate(_ptr(y), _ptr(z), y.size)
    if st != 0:
        raise RuntimeError(f"oracle_gate failed with status {st}")
    return y


def ss2d_forward(x, delta, A_log, Bs, Cs, Dskip, delta_bias, *, K=4,
                 bbar="euler", threads=1, return_dirs=False, z=None, _lib=None):
    """SS2D forward in float64.  x (B,D,H,W); delta (B,K,D,L); Bs, Cs
    (B,K,N,L); A_log (K*D,N); Dskip, delta_bias (K*D,).  Returns y (B,D,H,W)
    and, if asked, the per-direction outputs (B,K,D,L) in pixel order.  With
    z (the layout of x): the merged output times SiLU(z) (the per-direction
    outputs stay ungated)."""
    x = _f64(x)
    Bb, D, H, W = x.shape
    L = H * W
    delta, Bs, Cs = _f64(delta), _f64(Bs), _f64(Cs)
    A_log, Dskip, delta_bias = _f64(A_log), _f64(Dskip), _f64(delta_bias)
    N = Bs.shape[2]
    assert delta.shape == (Bb, K, D, L) and Bs.shape == (Bb, K, N, L)
    assert Cs.shape == Bs.shape and A_log.shape == (K * D, N)
    assert Dskip.shape == (K * D,) and delta_bias.shape == (K * D,)
    y = np.empty((Bb, D, H, W))
    yd = np.empty((Bb, K, D, L)) if return_dirs else None
    lb = _lib or lib()
    st = lb.oracle_ss2d_forward(_ptr(x), _ptr(delta), _ptr(A_log), _ptr(Bs),
                                _ptr(Cs), _ptr(Dskip), _ptr(delta_bias),
                                _ptr(y), _ptr(yd) if yd is not None else None,
                                Bb, D, H, W, N, K, _BBAR[bbar], int(threads))
    if st != 0:
        raise RuntimeError(f"oracle_ss2d_forward failed with status {st}")
    if z is not None:
        _gate(y, z, lb)
    return (y, yd) if return_dirs else y


def selective_scan_fwd(u, delta, A_log, Bs, Cs, Dskip, delta_bias, *, K=2,
                       bbar="euler", threads=1, return_dirs=False, z=None, _lib=None):
    """1D selective scan in float64: u (B,D,L); K=1 forward, K=2 forward plus
    reversed (flipped back, then added).  With z (B,D,L): the summed output
    times SiLU(z)."""
    u = _f64(u)
    Bb, D, L = u.shape
    delta, Bs, Cs = _f64(delta), _f64(Bs), _f64(Cs)
    A_log, Dskip, delta_bias = _f64(A_log), _f64(Dskip), _f64(delta_bias)
    N = Bs.shape[2]
    assert delta.shape == (Bb, K, D, L) and Bs.shape == (Bb, K, N, L)
    assert Cs.shape == Bs.shape and A_log.shape == (K * D, N)
    y = np.empty((Bb, D, L))
    yd = np.empty((Bb, K, D, L)) if return_dirs else None
    lb = _lib or lib()
    st = lb.oracle_selective_scan_fwd(_ptr(u), _ptr(delta), _ptr(A_log),
                                      _ptr(Bs), _ptr(Cs), _ptr(Dskip),
                                      _ptr(delta_bias), _ptr(y),
                                      _ptr(yd) if yd is not None else None,
                                      Bb, D, L, N, K, _BBAR[bbar],
                                      int(threads))
    if st != 0:
        raise RuntimeError(f"oracle_selective_scan_fwd failed with status {st}")
    if z is not None:
        _gate(y, z, lb)
    return (y, yd) if return_dirs else y


def softplus(z: float) -> float:
    return lib().oracle_softplus(float(z))


def silu(z: float) -> float:
    return lib().oracle_silu(float(z))


def scan_pixel(mode: int, k: int, l: int, H: int, W: int) -> int:
    return lib().oracle_scan_pixel(mode, k, l, H, W)


def max_threads() -> int:
    return lib().oracle_max_threads()


def front_scan(x, conv_w, conv_b, W_x, w_dt, A_log, Dskip, delta_bias, *, storage=None,
               operand="f64", threads=1):
    """The front of every direction (:func:`front_directions`) followed by
    that direction's selective scan over its own u, delta, B and C, each
    direction's output turned back to the sequence order (direction 1 is
    reversed) and the K outputs summed: y (B, D, L) float64.  A_log (K*D, N),
    Dskip and delta_bias (K*D,) as in :func:`selective_scan_fwd`."""
    u, delta, Bs, Cs = front_directions(x, conv_w, conv_b, W_x, w_dt, storage=storage,
                                        operand=operand)
    K, D = u.shape[1], u.shape[2]
    A_log = np.asarray(A_log, dtype=np.float64)
    Dskip = np.asarray(Dskip, dtype=np.float64)
    delta_bias = np.asarray(delta_bias, dtype=np.float64)
    y = None
    for k in range(K):
        rows = slice(k * D, (k + 1) * D)
        yk = selective_scan_fwd(u[:, k], delta[:, k:k + 1], A_log[rows], Bs[:, k:k + 1],
                                Cs[:, k:k + 1], Dskip[rows], delta_bias[rows], K=1,
                                threads=threads)
        if k == 1:
            yk = yk[:, :, ::-1]
        y = yk if y is None else y + yk
    return np.ascontiguousarray(y)

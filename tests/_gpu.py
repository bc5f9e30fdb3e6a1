"""Helpers shared by the GPU tests: move seeded workloads onto the device,
run the CUDA library through its binding, run the float64 oracle on the
same values, and compare under the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from selective_scan_ss2d_b200 import binding
from selective_scan_ss2d_b200 import workloads as wl

# fp32 inputs: per element |y - y_ref| <= FP32_TOL * max(1, |y_ref|)
FP32_TOL = 1e-4
# bf16 or fp16 inputs (fp32 state): ||y - y_ref||_2 <= BF16_REL_L2 * ||y_ref||_2
BF16_REL_L2 = 1e-3


def to_torch(a: np.ndarray, dtype: str, device) -> torch.Tensor:
    if a.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device) if device is not None else t


def tensors(inp: wl.Inputs, device="cuda", pin=False) -> dict:
    out = {}
    for name in wl.Inputs.STREAMED + wl.Inputs.PARAMS:
        t = to_torch(getattr(inp, name), inp.cfg.dtype, None)
        if device is None:
            out[name] = t.pin_memory() if pin else t.contiguous()
        else:
            out[name] = t.to(device)
    return out


def run_gpu(inp: wl.Inputs, variant: int = -1, device="cuda", t=None) -> np.ndarray:
    t = t if t is not None else tensors(inp, device)
    fn = binding.ss2d_forward if inp.cfg.kind == "2d" else binding.selective_scan_fwd
    y = fn(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"],
           variant=variant)
    if y.is_cuda:
        torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def run_oracle(inp: wl.Inputs, threads: int = 0) -> np.ndarray:
    f = inp.as_f64()
    th = threads or oracle.max_threads()
    if inp.cfg.kind == "2d":
        return oracle.ss2d_forward(f["x"], f["delta"], f["A_log"], f["Bs"], f["Cs"],
                                   f["Dskip"], f["delta_bias"], K=inp.cfg.K, threads=th)
    return oracle.selective_scan_fwd(f["x"], f["delta"], f["A_log"], f["Bs"], f["Cs"],
                                     f["Dskip"], f["delta_bias"], K=inp.cfg.K, threads=th)


def assert_close(y: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    if dtype == wl.F32:
        err = np.abs(y - ref)
        bound = FP32_TOL * np.maximum(1.0, np.abs(ref))
        worst = np.argmax(err / bound)
        assert np.all(err <= bound), (
            f"{what}: fp32 bound exceeded at flat index {worst}: "
            f"|{y.flat[worst]} - {ref.flat[worst]}| = {err.flat[worst]:.3e} "
            f"> {bound.flat[worst]:.3e}")
    else:
        rel = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300)
        assert rel <= BF16_REL_L2, f"{what}: relative L2 error {rel:.3e} > {BF16_REL_L2}"


def vary_params(inp: wl.Inputs, seed: int) -> wl.Inputs:
    """The same workload with per-row parameters that differ from row to row:
    A_log + U(-0.7, 0.7) per element and Dskip ~ U(0.3, 1.7) per row (the
    recipe's A_log rows are all ln(n + 1) and its Dskip all 1, which would
    hide a wrong row index)."""
    rng = np.random.default_rng([seed, 0xa1])
    A_log = (inp.A_log + rng.uniform(-0.7, 0.7, inp.A_log.shape)).astype(np.float32)
    Dskip = rng.uniform(0.3, 1.7, inp.Dskip.shape).astype(np.float32)
    return wl.Inputs(inp.cfg, inp.x, inp.delta, inp.Bs, inp.Cs, A_log, Dskip, inp.delta_bias)

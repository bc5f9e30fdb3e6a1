"""GPU parity of the fused front (causal depthwise conv1d + SiLU + x_proj on
the tensor cores + dt_proj, "Vision Mamba" tutorial SelectiveSSM and the Vim
block of "Vision Mamba ..." section 4.3) and of the front followed by the
scan, against the float64 oracle (``oracle.front_scan``,
``ss2d_front_np.front_directions``) on the same seeded inputs.

The oracle takes the library's precision readings: x_proj multiplies
bfloat16 operands (u and W_x rounded to nearest even) with exact sums, and
the scan reads u as stored in the input dtype.  Bars:
* y: relative L2 <= 1e-3 for every input dtype -- the bar of the bf16
  path, because x_proj's operands are bfloat16 whatever the input dtype
  (the float32 per-element bar of the plain scan does not apply: the
  kernel rounds its float32 u to bfloat16, the oracle its float64 u, and
  the rare value that sits between them on a rounding boundary moves one
  product of x_proj by 2^-8 of itself);
* the front's own outputs: u within one unit in the last place of its
  storage dtype; dt_raw, B, C within 1e-3 of sum_d |u_d| |W_d| (a wrong
  operand layout gives errors of order one);
* the bounded wait: a wait that nothing completes ends and is reported.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import _gpu
from oracle import ss2d_front_np
from selective_scan_ss2d_b200 import binding
from selective_scan_ss2d_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TORCH = {wl.F32: torch.float32, wl.BF16: torch.bfloat16, wl.F16: torch.float16}
STORAGE = {wl.F32: "f32", wl.BF16: "bf16", wl.F16: "f16"}


def make_front(B, L, D, N, K, dtype, seed):
    """The seeded front inputs (``workloads.make_front_inputs``) with x as the
    float32 values the GPU sees."""
    cfg = wl.FrontConfig(f"front_{B}_{L}_{D}_{N}_{K}", B, L, D, N, K, dtype)
    inp = wl.make_front_inputs(cfg, seed=seed)
    out = {n: getattr(inp, n) for n in wl.FrontInputs.WEIGHTS}
    out["x"] = inp.x_f64().astype(np.float32)
    return out


def to_dev(a, dtype):
    return {k: torch.from_numpy(v).to("cuda").to(TORCH[dtype] if k == "x" else torch.float32)
            for k, v in a.items()}


SHAPES = [  # B, L, D, N, K
    (2, 200, 96, 16, 2),     # two step tiles (ragged), a ragged channel block
    (1, 128, 64, 16, 1),     # one tile, one block
    (2, 197, 192, 16, 2),    # the Vim-S token count, three channel blocks
    (1, 300, 40, 8, 2),      # d_state 8, fewer channels than a block
    (2, 64, 70, 5, 1),       # odd N, a partial tile
    (1, 1100, 64, 16, 2),    # long enough to be chunked
    (2, 150, 130, 24, 2),    # two state groups, a 2-channel last tile
    (2, 199, 70, 16, 2),     # a last tile whose rows are not a whole number of float4
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_L{}_D{}_N{}_K{}".format(*s))
@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16, wl.F16])
def test_front_scan_matches_oracle(shape, dtype):
    B, L, D, N, K = shape
    a = make_front(B, L, D, N, K, dtype, seed=31)
    ref = oracle.front_scan(a["x"], a["conv_w"], a["conv_b"], a["W_x"], a["w_dt"], a["A_log"],
                            a["Dskip"], a["delta_bias"], storage=STORAGE[dtype],
                            operand="bf16", threads=oracle.max_threads())
    t = to_dev(a, dtype)
    y = binding.selective_scan_fwd_front(t["x"], t["conv_w"], t["conv_b"], t["W_x"], t["w_dt"],
                                         t["A_log"], t["Dskip"], t["delta_bias"])
    torch.cuda.synchronize()
    assert binding.ss2d_check_waits() == 0
    # the bf16-path bar for every dtype (x_proj runs on bf16 operands)
    _gpu.assert_close(y.cpu().numpy().astype(np.float64), ref, wl.BF16, f"front {shape}")


@pytest.mark.parametrize("shape", [(2, 200, 96, 16, 2), (1, 256, 192, 16, 1), (2, 64, 70, 5, 2)],
                         ids=lambda s: "B{}_L{}_D{}_N{}_K{}".format(*s))
@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16])
def test_front_projections_match_oracle(shape, dtype):
    B, L, D, N, K = shape
    L8 = (L + 7) // 8 * 8
    a = make_front(B, L8, D, N, K, dtype, seed=32)
    u_ref, delta_ref, B_ref, C_ref = ss2d_front_np.front_directions(
        a["x"], a["conv_w"], a["conv_b"], a["W_x"], a["w_dt"], storage=STORAGE[dtype],
        operand="bf16")
    t = to_dev(a, dtype)
    u, dt_raw, Bs, Cs = binding.ss2d_front_project(t["x"], t["conv_w"], t["conv_b"], t["W_x"])
    torch.cuda.synchronize()
    assert binding.ss2d_check_waits() == 0
    u = u.float().cpu().numpy().astype(np.float64)
    # u: the same rounding of a float32 and a float64 SiLU: equal but for the
    # rare value within float32 error of a rounding boundary
    # (float32: the kernel's SiLU uses the fast exp and division, a few
    # float32 ulp; the conv's cancellation near u = 0 is covered by 1e-6)
    rel = {wl.F32: 2e-6, wl.BF16: 2.0 ** -7, wl.F16: 2.0 ** -10}[dtype]
    assert np.all(np.abs(u - u_ref) <= rel * np.abs(u_ref) + 1e-6)
    # dt_raw, B, C against the scale of their sums
    x = a["x"].astype(np.float64)
    for k in range(K):
        seq = x if k == 0 else x[:, ::-1, :]
        uk = ss2d_front_np.silu(ss2d_front_np.causal_depthwise_conv(
            seq, a["conv_w"][k].astype(np.float64), a["conv_b"][k].astype(np.float64)))
        scale = np.abs(uk) @ np.abs(a["W_x"][k].astype(np.float64)).T   # (B, L, 1 + 2N)
        dt_ref = delta_ref[:, k, 0] / a["w_dt"][k, 0]
        got = dt_raw[:, k].cpu().numpy()
        assert np.all(np.abs(got - dt_ref) <= 1e-3 * scale[:, :, 0] + 1e-6), "dt_raw"
        for n in range(N):
            gb = Bs[:, k, n].cpu().numpy()
            gc = Cs[:, k, n].cpu().numpy()
            assert np.all(np.abs(gb - B_ref[:, k, n]) <= 1e-3 * scale[:, :, 1 + n] + 1e-6), "B"
            assert np.all(np.abs(gc - C_ref[:, k, n]) <= 1e-3 * scale[:, :, 1 + N + n] + 1e-6), "C"


def test_front_deterministic():
    a = make_front(2, 200, 96, 16, 2, wl.BF16, seed=33)
    t = to_dev(a, wl.BF16)
    args = [t[n] for n in ("x", "conv_w", "conv_b", "W_x", "w_dt", "A_log", "Dskip", "delta_bias")]
    y1 = binding.selective_scan_fwd_front(*args)
    y2 = binding.selective_scan_fwd_front(*args)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_front_more_sequences_than_one_grid_dimension():
    # B * K = 66000 (b, direction) pairs: more than a grid's y or z dimension holds
    B, L, D, N, K = 33000, 3, 2, 2, 2
    a = make_front(B, L, D, N, K, wl.BF16, seed=36)
    ref = oracle.front_scan(a["x"], a["conv_w"], a["conv_b"], a["W_x"], a["w_dt"], a["A_log"],
                            a["Dskip"], a["delta_bias"], storage=STORAGE[wl.BF16],
                            operand="bf16", threads=oracle.max_threads())
    t = to_dev(a, wl.BF16)
    y = binding.selective_scan_fwd_front(t["x"], t["conv_w"], t["conv_b"], t["W_x"], t["w_dt"],
                                         t["A_log"], t["Dskip"], t["delta_bias"])
    torch.cuda.synchronize()
    assert binding.ss2d_check_waits() == 0
    _gpu.assert_close(y.cpu().numpy().astype(np.float64), ref, wl.BF16, "front B*K > 65535")


def test_front_rejects_bad_arguments():
    a = make_front(1, 64, 64, 4, 2, wl.F32, seed=34)
    t = to_dev(a, wl.F32)
    with pytest.raises(ValueError):
        binding.selective_scan_fwd_front(t["x"].cpu(), t["conv_w"], t["conv_b"], t["W_x"],
                                         t["w_dt"], t["A_log"], t["Dskip"], t["delta_bias"])
    with pytest.raises(ValueError):
        binding.selective_scan_fwd_front(t["x"], t["conv_w"][:, :, :3].contiguous(), t["conv_b"],
                                         t["W_x"], t["w_dt"], t["A_log"], t["Dskip"],
                                         t["delta_bias"])
    lib = binding.lib()
    p = [binding._ptr(t[n]) for n in ("x", "conv_w", "conv_b", "W_x", "w_dt", "A_log", "Dskip",
                                      "delta_bias")]
    y = torch.empty((1, 64, 64), device="cuda")
    assert lib.selective_scan_fwd_front(*p, binding._ptr(y), 1, 64, 64, 4, 3, 0, None) == -4
    assert lib.selective_scan_fwd_front(*p, binding._ptr(y), 1, 64, 64, 65, 2, 0, None) == -5
    assert lib.selective_scan_fwd_front(*p, None, 1, 64, 64, 4, 2, 0, None) == -1


def test_bounded_wait_runs_out_and_is_reported():
    """A wait that nothing can complete ends after its limit; the fault is
    reported once, and the context stays usable."""
    assert binding.ss2d_check_waits() == 0
    binding.ss2d_wait_selftest(2000)   # 2 ms
    torch.cuda.synchronize()
    assert binding.ss2d_check_waits() == -8
    assert "bounded wait" in binding.lib().ss2d_last_error().decode()
    assert binding.ss2d_check_waits() == 0
    # the device still runs work
    a = make_front(1, 128, 64, 16, 1, wl.BF16, seed=35)
    t = to_dev(a, wl.BF16)
    y = binding.selective_scan_fwd_front(*[t[n] for n in ("x", "conv_w", "conv_b", "W_x", "w_dt",
                                                          "A_log", "Dskip", "delta_bias")])
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    assert binding.ss2d_check_waits() == 0

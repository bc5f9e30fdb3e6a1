"""GPU parity: the CUDA library against the float64 oracle on the same seeded
inputs, through the C ABI (ctypes binding).

Bars: index maps bit-exact (integer-valued inputs); fp32 inputs per element
|y - y_ref| <= 1e-4 * max(1, |y_ref|); bf16 or fp16 inputs (fp32 state)
relative L2 <= 1e-3, the oracle reading the same rounded values.
"""
import numpy as np
import pytest
import torch

import oracle
import _gpu
from selective_scan_ss2d_b200 import binding
from selective_scan_ss2d_b200 import workloads as wl

pytestmark = pytest.mark.gpu

NV = None


def nvariants():
    global NV
    if NV is None:
        NV = binding.ss2d_num_variants()
    return NV


def small(kind="2d", B=2, D=12, H=7, W=9, K=4, N=16, dtype=wl.F32):
    if kind == "1d":
        return wl.Config(f"small1d_{B}_{D}_{W}_{K}_{N}_{dtype}", "1d", B, D, 1, W, K, N, dtype)
    return wl.Config(f"small2d_{B}_{D}_{H}x{W}_{K}_{N}_{dtype}", "2d", B, D, H, W, K, N, dtype)


# ---------------------------------------------------------------------------
# small shapes: several tiles, ragged tails, every variant
# ---------------------------------------------------------------------------
SMALL_2D = [
    small(),                                        # non-square, L = 63 (ragged)
    small(B=2, D=40, H=14, W=14, K=4, N=16),        # VMamba-B stage-3 image, two column wraps
    small(B=1, D=24, H=11, W=23, K=4, N=16),        # odd height between 8 and 16
    small(B=1, D=8, H=8, W=8, K=4, N=4),            # the tiny config's shape
    small(B=3, D=37, H=5, W=13, K=4, N=16),         # D not a multiple of any tile
    small(B=2, D=16, H=16, W=20, K=4, N=8),         # L = 320 (> one chunk)
    small(B=1, D=8, H=33, W=31, K=4, N=16),         # L = 1023, long ragged chunks
    small(B=2, D=9, H=6, W=5, K=2, N=5),            # K = 2, odd N
    small(B=2, D=9, H=6, W=5, K=1, N=1),            # K = 1, N = 1
    small(B=1, D=40, H=24, W=16, K=4, N=16),        # D = 32 + 8, 384 steps
    small(B=2, D=8, H=56, W=16, K=4, N=5),          # VMamba-T's image height, odd N
    small(B=1, D=33, H=32, W=8, K=4, N=16),         # tall and narrow
]
SMALL_1D = [
    small("1d", B=3, D=20, W=197, K=2, N=16),
    small("1d", B=2, D=7, W=50, K=1, N=3),
    small("1d", B=1, D=33, W=1000, K=2, N=16),
]


@pytest.mark.parametrize("cfg", SMALL_2D + SMALL_1D, ids=lambda c: c.name)
@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16, wl.F16])
def test_small_shapes_all_variants(cfg, dtype):
    cfg = cfg.with_(dtype=dtype)
    inp = wl.make_inputs(cfg, seed=1)
    ref = _gpu.run_oracle(inp)
    t = _gpu.tensors(inp)
    for v in [-1] + list(range(nvariants())):
        y = _gpu.run_gpu(inp, variant=v, t=t)
        _gpu.assert_close(y, ref, dtype, f"{cfg.name} variant {v}")


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_config(seed):
    inp = wl.make_inputs("tiny_fp32", seed=seed)
    y = _gpu.run_gpu(inp)
    _gpu.assert_close(y, _gpu.run_oracle(inp), wl.F32, "tiny_fp32")


# ---------------------------------------------------------------------------
# index maps: bit-exact with integer-valued inputs
# ---------------------------------------------------------------------------
def _running_sum_inputs(cfg, rng):
    """dt = 32 exactly (softplus(z) = z above 20), A = 0 (A_log = -inf), N = 1,
    B = 1, C = 1/32: every direction's output is the running sum of the
    integer inputs along its scan order, exact in float32."""
    K, D, L = cfg.K, cfg.D, cfg.L
    xshape = (cfg.B, D, cfg.H, cfg.W) if cfg.kind == "2d" else (cfg.B, D, L)
    x = rng.integers(-4, 5, size=xshape).astype(np.float32)
    return wl.Inputs(cfg, x,
                     np.zeros((cfg.B, K, D, L), np.float32),
                     np.ones((cfg.B, K, 1, L), np.float32),
                     np.full((cfg.B, K, 1, L), 1.0 / 32.0, np.float32),
                     np.full((K * D, 1), -np.inf, np.float32),
                     np.zeros(K * D, np.float32),
                     np.full(K * D, 32.0, np.float32))


# heights below 8 use the pixel walker; 8..15 can wrap a column twice within
# one 16-step sub-chunk, 16 and more at most once; odd 1D lengths take the
# realigned 4-byte loads of bf16 rows
INDEX_SHAPES = [small(B=2, D=5, H=5, W=7, N=1), small(B=1, D=3, H=56, W=56, N=1),
                small(B=1, D=2, H=24, W=40, N=1), small(B=1, D=4, H=7, W=9, K=2, N=1),
                small(B=1, D=3, H=14, W=14, N=1), small(B=1, D=2, H=9, W=17, N=1),
                small(B=1, D=2, H=11, W=6, N=1), small(B=1, D=2, H=16, W=3, N=1),
                small(B=1, D=2, H=15, W=33, N=1),
                small("1d", B=2, D=5, W=197, K=2, N=1), small("1d", B=2, D=3, W=201, K=2, N=1),
                small("1d", B=3, D=2, W=34, K=2, N=1)]


@pytest.mark.parametrize("cfg", INDEX_SHAPES, ids=lambda c: c.name)
@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16, wl.F16])
def test_index_maps_bit_exact(cfg, dtype):
    rng = np.random.default_rng(5)
    inp = _running_sum_inputs(cfg, rng)
    if dtype != wl.F32:
        # every value involved (small integers, 0, 1, 1/32) is exact in bf16 and f16
        cast = wl.f32_to_bf16_bits if dtype == wl.BF16 else (lambda a: a.astype(np.float16))
        inp = wl.Inputs(inp.cfg.with_(dtype=dtype), cast(inp.x), cast(inp.delta), cast(inp.Bs),
                        cast(inp.Cs), inp.A_log, inp.Dskip, inp.delta_bias)
    # The exact result is an integer running sum.  The oracle's float64
    # softplus(32) is 32 * (1 + 4e-16), so its sums carry residues below
    # 1e-12; rounding to the nearest integer recovers the exact values.
    ref64 = _gpu.run_oracle(inp)
    ref = np.rint(ref64)
    assert np.abs(ref64 - ref).max() < 1e-9
    ref = ref.astype(np.float32)
    t = _gpu.tensors(inp)
    for v in [-1] + list(range(nvariants())):
        y = _gpu.run_gpu(inp, variant=v, t=t).astype(np.float32)
        assert np.array_equal(y, ref), f"variant {v}: index maps not bit-exact"


def test_identity_scan_is_4x_bit_exact():
    cfg = small(B=2, D=10, H=9, W=11, N=16)
    rng = np.random.default_rng(6)
    inp = wl.make_inputs(cfg, seed=2)
    inp.x = rng.integers(-100, 101, size=inp.x.shape).astype(np.float32)
    inp.Bs = np.zeros_like(inp.Bs)
    y = _gpu.run_gpu(inp).astype(np.float32)
    assert np.array_equal(y, 4.0 * inp.x)


# ---------------------------------------------------------------------------
# determinism, host-buffer path, errors
# ---------------------------------------------------------------------------
def test_deterministic():
    inp = wl.make_inputs(small(B=2, D=24, H=14, W=14, dtype=wl.BF16), seed=3)
    t = _gpu.tensors(inp)
    for v in [-1] + list(range(nvariants())):
        a = _gpu.run_gpu(inp, variant=v, t=t)
        b = _gpu.run_gpu(inp, variant=v, t=t)
        assert np.array_equal(a, b)


@pytest.mark.parametrize("pin", [False, True])
def test_host_buffers_match_device(pin):
    inp = wl.make_inputs(small(B=2, D=16, H=10, W=12, dtype=wl.BF16), seed=4)
    yd = _gpu.run_gpu(inp)
    th = _gpu.tensors(inp, device=None, pin=pin)
    yh = binding.ss2d_forward(th["x"], th["delta"], th["A_log"], th["Bs"], th["Cs"],
                              th["Dskip"], th["delta_bias"])
    assert not yh.is_cuda
    assert np.array_equal(yh.numpy().astype(np.float64), yd)


# the host path cuts a batch with more than 16 MB of input into slices
# whose copies overlap the scans of the others; each slice keeps the whole
# call's chunk plan, so the bits are the device path's: uneven slices,
# chunked and unchunked, K = 4, K = 2 (added into y) and the 1D call
@pytest.mark.parametrize("case", [
    ("2d", 5, 128, 64, 64, 4, 16, wl.BF16),   # 30 MB: slices of 2 and 3 elements
    ("2d", 3, 64, 96, 96, 4, 16, wl.F32),     # chunked rows, 3 slices of one
    ("2d", 7, 256, 48, 48, 2, 8, wl.F16),     # K = 2: slices of 3 and 4
    ("1d", 40, 768, 1, 197, 2, 16, wl.BF16),  # the 1D bidirectional call, 3 slices
    ("1d", 6, 512, 1, 1100, 2, 33, wl.BF16),  # two state groups, chunked, 2 slices
    ("2d", 3, 16, 10, 12, 4, 16, wl.BF16),    # under 16 MB: one piece
], ids=lambda c: "{}_B{}_D{}_{}x{}_K{}_N{}_{}".format(*c))
def test_host_slices_match_device(case):
    kind, B, D, H, W, K, N, dt = case
    cfg = (wl.Config(f"hs_{B}_{D}_{W}_{K}_{N}_{dt}", "1d", B, D, 1, W, K, N, dt) if kind == "1d"
           else wl.Config(f"hs_{B}_{D}_{H}x{W}_{K}_{N}_{dt}", "2d", B, D, H, W, K, N, dt))
    inp = wl.make_inputs(cfg, seed=11)
    yd = _gpu.run_gpu(inp)
    th = _gpu.tensors(inp, device=None, pin=True)
    fn = binding.ss2d_forward if kind == "2d" else binding.selective_scan_fwd
    yh = fn(th["x"], th["delta"], th["A_log"], th["Bs"], th["Cs"], th["Dskip"], th["delta_bias"])
    assert not yh.is_cuda
    assert np.array_equal(yh.numpy().astype(np.float64), yd)


def test_mixed_pointers_rejected():
    inp = wl.make_inputs(small(B=1, D=4, H=4, W=4), seed=0)
    t = _gpu.tensors(inp)
    xc = t["x"].cpu()
    lib = binding.lib()
    args = [binding._ptr(a) for a in (xc, t["delta"], t["A_log"], t["Bs"], t["Cs"],
                                      t["Dskip"], t["delta_bias"])]
    y = torch.empty_like(t["x"], dtype=torch.float32)
    rc = lib.ss2d_forward(*args, binding._ptr(y), 1, 4, 4, 4, 16, 4, 0, None)
    assert rc == -9


def test_empty_shapes():
    x = torch.zeros(0, 4, 3, 3, device="cuda")
    delta = torch.zeros(0, 4, 4, 9, device="cuda")
    Bs = torch.zeros(0, 4, 16, 9, device="cuda")
    A_log = torch.zeros(16, 16, device="cuda")
    Dk = torch.zeros(16, device="cuda")
    y = binding.ss2d_forward(x, delta, A_log, Bs, Bs, Dk, Dk)
    assert y.shape == (0, 4, 3, 3)


def test_extreme_delta():
    """softplus saturation and underflow: dt far above 20 and far below."""
    cfg = small(B=1, D=6, H=5, W=6, N=16)
    inp = wl.make_inputs(cfg, seed=7)
    inp.delta = (inp.delta * 30.0).astype(np.float32)
    _gpu.assert_close(_gpu.run_gpu(inp), _gpu.run_oracle(inp), wl.F32, "extreme delta")


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration the benchmark times:
# sampled output channels against the oracle run channel by channel
# ---------------------------------------------------------------------------
FULL = ["tiny_fp32", "vmamba_t_stage1", "vmamba_b_stage3", "highres_256", "vim_s_bidir"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_channels(name):
    cfg = wl.CONFIGS[name]
    inp = wl.make_inputs(cfg, seed=0)
    y = _gpu.run_gpu(inp)
    rng = np.random.default_rng(123)
    pairs = {(0, 0), (cfg.B - 1, cfg.D - 1)}
    while len(pairs) < min(8, cfg.B * cfg.D):
        pairs.add((int(rng.integers(cfg.B)), int(rng.integers(cfg.D))))
    got, want = [], []
    for (b, d) in sorted(pairs):
        sub = wl.channel_subproblem(inp, b, d)
        want.append(_gpu.run_oracle(sub)[0, 0].reshape(-1))
        got.append(y[b, d].reshape(-1))
    _gpu.assert_close(np.concatenate(got), np.concatenate(want), cfg.dtype, name)


# ---------------------------------------------------------------------------
# per-direction outputs and the timed call
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("cfg", [small(B=2, D=40, H=7, W=9, K=4), small(B=1, D=33, H=20, W=12, K=2),
                                 small("1d", B=2, D=33, W=100, K=2)],
                         ids=lambda c: c.name)
def test_scan_directions_match_oracle(cfg):
    inp = wl.make_inputs(cfg, seed=8)
    f = inp.as_f64()
    fn = oracle.ss2d_forward if cfg.kind == "2d" else oracle.selective_scan_fwd
    _, yd_ref = fn(f["x"], f["delta"], f["A_log"], f["Bs"], f["Cs"], f["Dskip"],
                   f["delta_bias"], K=cfg.K, return_dirs=True)
    t = _gpu.tensors(inp)
    for v in [-1, 3, 5]:
        yd = binding.ss2d_scan_directions(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"],
                                          t["Dskip"], t["delta_bias"], two_d=cfg.kind == "2d",
                                          variant=v)
        torch.cuda.synchronize()
        got = yd.double().cpu().numpy().reshape(cfg.B, cfg.K, cfg.D, cfg.L)
        _gpu.assert_close(got, yd_ref, wl.F32, f"directions variant {v}")


@pytest.mark.parametrize("cfg", [small(B=2, D=40, H=20, W=12, K=2, dtype=wl.BF16),
                                 small("1d", B=3, D=70, W=197, K=2),
                                 small("1d", B=1, D=33, W=1100, K=2, dtype=wl.BF16)],
                         ids=lambda c: c.name)
def test_two_directions_added_in_the_scan_equal_their_sum(cfg):
    # K = 2 with N <= 16: the output pass adds both directions into y; two
    # float32 terms meet in either order with the same bits, so y is exactly
    # the float32 sum of the per-direction outputs
    inp = wl.make_inputs(cfg, seed=12)
    t = _gpu.tensors(inp)
    lane = [i for i in range(nvariants()) if binding.ss2d_variant_name(i) == "lane2_wave"]
    for v in [-1, 3, 5] + lane:
        y = _gpu.run_gpu(inp, variant=v, t=t)
        yd = binding.ss2d_scan_directions(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"],
                                          t["Dskip"], t["delta_bias"], two_d=cfg.kind == "2d",
                                          variant=v)
        torch.cuda.synchronize()
        d = yd.cpu().numpy().reshape(cfg.B, cfg.K, cfg.D, cfg.L)
        want = (d[:, 0] + d[:, 1]).astype(np.float32).reshape(inp.x.shape)
        assert np.array_equal(y.astype(np.float32), want), f"variant {v}"


def test_timed_call_matches_forward():
    cfg = small(B=2, D=70, H=24, W=40, K=4, dtype=wl.BF16)
    inp = wl.make_inputs(cfg, seed=9)
    t = _gpu.tensors(inp)
    for v in [-1, 3]:
        y1 = _gpu.run_gpu(inp, variant=v, t=t)
        y2 = torch.empty(inp.x.shape, dtype=torch.float32, device="cuda")
        ms = binding.ss2d_forward_timed(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"],
                                        t["Dskip"], t["delta_bias"], y2, variant=v)
        assert np.array_equal(y2.double().cpu().numpy(), y1)
        plan = binding.ss2d_plan(True, cfg.B, cfg.D, cfg.H, cfg.W, cfg.N, cfg.K, v)
        assert ms[2] > 0 and ms[3] > 0
        assert (ms[0] > 0) == (plan["num_chunks"] > 1)


# ---------------------------------------------------------------------------
# the SiLU output gate (gated entry points)
# ---------------------------------------------------------------------------
GATED = [small(B=2, D=12, H=7, W=9, K=4, N=16), small(B=1, D=40, H=14, W=14, K=4, N=16),
         small(B=1, D=16, H=20, W=24, K=2, N=16), small(B=2, D=9, H=6, W=5, K=1, N=5),
         small(B=1, D=8, H=40, W=40, K=4, N=16),
         small("1d", B=3, D=20, W=197, K=2, N=16), small("1d", B=2, D=16, W=64, K=2, N=16),
         small("1d", B=2, D=7, W=50, K=1, N=3)]


@pytest.mark.parametrize("cfg", GATED, ids=lambda c: c.name)
@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16, wl.F16])
def test_gated_matches_oracle(cfg, dtype):
    cfg = cfg.with_(dtype=dtype)
    inp = wl.make_inputs(cfg, seed=4)
    zraw = wl.make_gate(cfg, seed=4)
    f = inp.as_f64()
    z64 = wl.gate_as_f64(zraw, cfg)
    th = oracle.max_threads()
    if cfg.kind == "2d":
        ref = oracle.ss2d_forward(f["x"], f["delta"], f["A_log"], f["Bs"], f["Cs"], f["Dskip"],
                                  f["delta_bias"], K=cfg.K, threads=th, z=z64)
    else:
        ref = oracle.selective_scan_fwd(f["x"], f["delta"], f["A_log"], f["Bs"], f["Cs"],
                                        f["Dskip"], f["delta_bias"], K=cfg.K, threads=th, z=z64)
    t = _gpu.tensors(inp)
    z = _gpu.to_torch(zraw, cfg.dtype, "cuda")
    fn = binding.ss2d_forward_gated if cfg.kind == "2d" else binding.selective_scan_fwd_gated
    y = fn(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"], z)
    torch.cuda.synchronize()
    _gpu.assert_close(y.cpu().numpy().astype(np.float64), ref, dtype, cfg.name + " gated")


def test_gated_rejects_host_pointers_and_missing_gate():
    inp = wl.make_inputs(small(B=1, D=4, H=4, W=4, K=4, N=4), seed=0)
    t = _gpu.tensors(inp, device=None)
    z = torch.zeros_like(t["x"])
    with pytest.raises(binding.SS2DError) as ei:
        binding.ss2d_forward_gated(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"],
                                   t["delta_bias"], z)
    assert ei.value.status == -9
    lib = binding.lib()
    td = _gpu.tensors(inp)
    y = torch.empty_like(td["x"])
    rc = lib.ss2d_forward_gated(*[binding._ptr(td[n]) for n in ("x", "delta", "A_log", "Bs", "Cs",
                                                               "Dskip", "delta_bias")],
                                None, binding._ptr(y), 1, 4, 4, 4, 4, 4, 0, None)
    assert rc == -1


# ---------------------------------------------------------------------------
# final states (ss2d_forward_final_state / selective_scan_fwd_final_state)
# ---------------------------------------------------------------------------
FINAL = [small(B=2, D=12, H=7, W=9), small(B=1, D=40, H=14, W=14), small(B=1, D=8, H=33, W=31),
         small(B=2, D=9, H=6, W=5, K=2, N=5), small(B=2, D=9, H=6, W=5, K=1, N=1),
         small("1d", B=3, D=20, W=197, K=2), small("1d", B=1, D=33, W=1000, K=2),
         small("1d", B=2, D=7, W=50, K=1, N=3)]


def _final_oracle(inp):
    f = inp.as_f64()
    return oracle.final_states(f["x"], f["delta"], f["A_log"], f["Bs"], f["delta_bias"],
                               K=inp.cfg.K, two_d=inp.cfg.kind == "2d")


@pytest.mark.parametrize("cfg", FINAL, ids=lambda c: c.name)
@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16])
def test_final_state_matches_oracle(cfg, dtype):
    cfg = cfg.with_(dtype=dtype)
    inp = wl.make_inputs(cfg, seed=6)
    ref = _final_oracle(inp)
    t = _gpu.tensors(inp)
    args = [t[n] for n in ("x", "delta", "A_log", "Bs", "Cs", "Dskip", "delta_bias")]
    for v in [-1] + list(range(nvariants())):
        y, h = binding.forward_final_state(*args, variant=v)
        torch.cuda.synchronize()
        # the same kernels as the plain forward: y identical to the bit
        y0 = _gpu.run_gpu(inp, variant=v, t=t)
        assert np.array_equal(y.cpu().numpy().astype(np.float64), y0), f"variant {v}: y differs"
        _gpu.assert_close(h.cpu().numpy().astype(np.float64), ref, dtype,
                          f"{cfg.name} variant {v} final state")


@pytest.mark.parametrize("name", ["vmamba_t_stage1", "highres_256"])
def test_final_state_full_size_sampled(name):
    inp = wl.make_inputs(name, seed=0)
    t = _gpu.tensors(inp)
    _, h = binding.forward_final_state(*[t[n] for n in ("x", "delta", "A_log", "Bs", "Cs", "Dskip",
                                                        "delta_bias")])
    h = h.cpu().numpy().astype(np.float64)
    for (b, d) in [(0, 0), (inp.cfg.B - 1, inp.cfg.D - 1), (0, inp.cfg.D // 2)]:
        sub = wl.channel_subproblem(inp, b, d)
        ref = _final_oracle(sub)
        _gpu.assert_close(h[b:b + 1, :, d:d + 1], ref, inp.cfg.dtype, f"{name} ({b},{d})")


def test_final_state_rejects_missing_or_host_buffers():
    inp = wl.make_inputs(small(B=1, D=4, H=4, W=4, K=4, N=4), seed=0)
    td = _gpu.tensors(inp)
    lib = binding.lib()
    names = ("x", "delta", "A_log", "Bs", "Cs", "Dskip", "delta_bias")
    y = torch.empty_like(td["x"])
    rc = lib.ss2d_forward_final_state(*[binding._ptr(td[n]) for n in names], binding._ptr(y),
                                      None, 1, 4, 4, 4, 4, 4, 0, None, -1)
    assert rc == -1
    hh = torch.empty((1, 4, 4, 4))
    rc = lib.ss2d_forward_final_state(*[binding._ptr(td[n]) for n in names], binding._ptr(y),
                                      binding._ptr(hh), 1, 4, 4, 4, 4, 4, 0, None, -1)
    assert rc == -9


# ---------------------------------------------------------------------------
# more than 16 states: groups of 16 run one after the other
# ---------------------------------------------------------------------------
WIDE_N = [small(B=2, D=12, H=7, W=9, N=17), small(B=1, D=40, H=14, W=14, N=32),
          small(B=1, D=8, H=33, W=31, N=40), small(B=2, D=9, H=6, W=5, K=2, N=64),
          small("1d", B=3, D=20, W=197, K=2, N=24), small("1d", B=2, D=7, W=50, K=1, N=48)]


@pytest.mark.parametrize("cfg", WIDE_N, ids=lambda c: c.name)
@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16])
def test_more_than_16_states(cfg, dtype):
    cfg = cfg.with_(dtype=dtype)
    inp = wl.make_inputs(cfg, seed=8)
    ref = _gpu.run_oracle(inp)
    href = _final_oracle(inp)
    t = _gpu.tensors(inp)
    args = [t[n] for n in ("x", "delta", "A_log", "Bs", "Cs", "Dskip", "delta_bias")]
    for v in [-1] + list(range(nvariants())):
        _gpu.assert_close(_gpu.run_gpu(inp, variant=v, t=t), ref, dtype, f"{cfg.name} v{v}")
        y, h = binding.forward_final_state(*args, variant=v)
        torch.cuda.synchronize()
        _gpu.assert_close(h.cpu().numpy().astype(np.float64), href, dtype,
                          f"{cfg.name} v{v} final state")


def test_more_than_16_states_full_size_sampled():
    """VMamba-T stage 1 with N = 32: sampled channels against the oracle."""
    cfg = wl.CONFIGS["vmamba_t_stage1"].with_(N=32)
    inp = wl.make_inputs(cfg, seed=0)
    y = _gpu.run_gpu(inp)
    for (b, d) in [(0, 0), (7, 191), (3, 77)]:
        sub = wl.channel_subproblem(inp, b, d)
        _gpu.assert_close(y[b:b + 1, d:d + 1], _gpu.run_oracle(sub), cfg.dtype, f"N=32 ({b},{d})")


VARIED = [small(B=2, D=40, H=7, W=9), small(B=1, D=24, H=14, W=14, K=2),
          small(B=1, D=8, H=33, W=31, N=24), small(B=2, D=9, H=6, W=5, K=1, N=8),
          small("1d", B=3, D=20, W=197, K=2), small("1d", B=2, D=7, W=50, K=1, N=40)]


@pytest.mark.parametrize("cfg", VARIED, ids=lambda c: c.name)
def test_row_parameters_are_read_per_row(cfg):
    """A_log and Dskip different in every row (k, d): every variant, final
    states included, against the oracle."""
    inp = _gpu.vary_params(wl.make_inputs(cfg, seed=12), seed=12)
    ref = _gpu.run_oracle(inp)
    href = _final_oracle(inp)
    t = _gpu.tensors(inp)
    args = [t[n] for n in ("x", "delta", "A_log", "Bs", "Cs", "Dskip", "delta_bias")]
    for v in [-1] + list(range(nvariants())):
        _gpu.assert_close(_gpu.run_gpu(inp, variant=v, t=t), ref, cfg.dtype, f"{cfg.name} v{v}")
        _, h = binding.forward_final_state(*args, variant=v)
        torch.cuda.synchronize()
        _gpu.assert_close(h.cpu().numpy().astype(np.float64), href, cfg.dtype,
                          f"{cfg.name} v{v} final state")


@pytest.mark.parametrize("name", ["vmamba_t_stage1", "vim_s_bidir"])
def test_eight_states_full_size_sampled(name):
    """d_state 8 ("VMamba架构解析", section 5) at full size: the 8-state
    kernels against the oracle on sampled channels."""
    cfg = wl.CONFIGS[name].with_(N=8)
    inp = wl.make_inputs(cfg, seed=0)
    y = _gpu.run_gpu(inp)
    for (b, d) in [(0, 0), (cfg.B - 1, cfg.D - 1), (cfg.B // 2, 77)]:
        sub = wl.channel_subproblem(inp, b, d)
        _gpu.assert_close(y[b:b + 1, d:d + 1], _gpu.run_oracle(sub), cfg.dtype, f"N=8 ({b},{d})")


# ---------------------------------------------------------------------------
# shapes past the launch limits of a single grid: more (b, chunk) pairs than
# a grid dimension holds, and maps too wide for the band-form merge
# ---------------------------------------------------------------------------
def test_more_chunk_launches_than_one_grid_dimension():
    """1D, B = 300, L = 4096 with 16-step chunks: 300 * 256 (b, chunk) pairs,
    more than 65535, run by looping over grid z."""
    cfg = small("1d", B=300, D=1, W=4096, K=1, N=4)
    inp = wl.make_inputs(cfg, seed=13)
    v = [i for i in range(nvariants()) if binding.ss2d_variant_name(i) == "wc2_lc16"][0]
    plan = binding.ss2d_plan(False, cfg.B, cfg.D, 1, cfg.L, cfg.N, cfg.K, v)
    assert cfg.B * plan["num_chunks"] > 65535
    _gpu.assert_close(_gpu.run_gpu(inp, variant=v), _gpu.run_oracle(inp), wl.F32, cfg.name)


def test_wide_map_plain_merge():
    """An 8 x 1600 map (K = 4): too wide for the band merge's tiles, merged
    one pixel per thread; every element against the oracle."""
    cfg = small(B=1, D=4, H=8, W=1600, K=4, N=16)
    inp = wl.make_inputs(cfg, seed=14)
    _gpu.assert_close(_gpu.run_gpu(inp), _gpu.run_oracle(inp), wl.F32, cfg.name)


def test_map_1024x1024_sampled_channels():
    """A 1024 x 1024 map, D = 8, bf16 (L = 2^20): sampled channels against the
    oracle."""
    cfg = small(B=1, D=8, H=1024, W=1024, K=4, N=16, dtype=wl.BF16)
    inp = wl.make_inputs(cfg, seed=15)
    y = _gpu.run_gpu(inp)
    for d in (0, 5):
        sub = wl.channel_subproblem(inp, 0, d)
        _gpu.assert_close(y[0:1, d:d + 1], _gpu.run_oracle(sub), wl.BF16, f"1024^2 d={d}")


@pytest.mark.parametrize("chunks", [4, 21, 101, 601, 1001])
def test_carry_segments(chunks):
    """The carry scan's segment plans, 16-step chunks (1D, K = 2, N = 5 so
    that threads of states past N idle): 3 chunk boundaries (16 rows per CTA,
    one segment each), 20 (two segments), 100 (eight), 600 (16 segments of
    38 chunks, one row per CTA), all staged in shared memory; 1000 (too long
    to stage: 32 segments read from global memory); every element against
    the oracle at the float32 bar."""
    cfg = small("1d", B=2, D=3, W=16 * chunks - 5, K=2, N=5)
    inp = wl.make_inputs(cfg, seed=16)
    v = [i for i in range(nvariants()) if binding.ss2d_variant_name(i) == "wc2_lc16"][0]
    plan = binding.ss2d_plan(False, cfg.B, cfg.D, 1, cfg.L, cfg.N, cfg.K, v)
    assert plan["num_chunks"] == chunks
    _gpu.assert_close(_gpu.run_gpu(inp, variant=v), _gpu.run_oracle(inp), wl.F32, cfg.name)

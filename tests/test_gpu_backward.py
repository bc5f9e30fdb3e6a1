"""Parity of the CUDA backward (ss2d_backward / selective_scan_bwd) with the
float64 backward oracle, on the same seeded inputs and cotangent.

Bar (every input dtype; the oracle reads the same rounded input values, so
the difference is float32 arithmetic only): per element of every gradient
array G, |G - G_ref| <= 1e-4 * (|G_ref| + rms(G_ref)).  The array's RMS
stands in for the forward's floor of 1 because gradient arrays have no
natural unit scale (dA_log is small when dt is, dBs large when D is)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import _gpu
from selective_scan_ss2d_b200 import binding
from selective_scan_ss2d_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GRAD_TOL = 1e-4
GRADS = binding.GRAD_NAMES


def small(kind="2d", B=2, D=12, H=7, W=9, K=4, N=16, dtype=wl.F32):
    if kind == "1d":
        return wl.Config(f"bwd1d_{B}_{D}_{W}_{K}_{N}_{dtype}", "1d", B, D, 1, W, K, N, dtype)
    return wl.Config(f"bwd2d_{B}_{D}_{H}x{W}_{K}_{N}_{dtype}", "2d", B, D, H, W, K, N, dtype)


def oracle_backward(inp, dy):
    f = inp.as_f64()
    fn = oracle.ss2d_backward if inp.cfg.kind == "2d" else oracle.selective_scan_bwd
    return fn(f["x"], f["delta"], f["A_log"], f["Bs"], f["Cs"], f["Dskip"], f["delta_bias"],
              dy.astype(np.float64), K=inp.cfg.K)


def gpu_backward(inp, dy, t=None):
    t = t if t is not None else _gpu.tensors(inp)
    fn = binding.ss2d_backward if inp.cfg.kind == "2d" else binding.selective_scan_bwd
    g = fn(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"],
           torch.from_numpy(dy).cuda())
    torch.cuda.synchronize()
    return {n: v.cpu().numpy().astype(np.float64) for n, v in g.items()}


def assert_grads_close(got, ref, what, names=GRADS):
    for n in names:
        a, r = got[n], ref[n]
        assert a.shape == r.shape, (what, n, a.shape, r.shape)
        assert np.all(np.isfinite(a)), f"{what}: {n} not finite"
        rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
        bound = GRAD_TOL * (np.abs(r) + rms)
        err = np.abs(a - r)
        if not np.all(err <= bound):
            i = int(np.argmax(err / np.maximum(bound, 1e-300)))
            raise AssertionError(f"{what}: {n} off at flat index {i}: got {a.flat[i]:.6e}, "
                                 f"oracle {r.flat[i]:.6e}, bound {bound.flat[i]:.3e} (rms {rms:.3e})")


SHAPES = [
    small(),                                         # L = 63: four chunks, ragged last one
    small(B=2, D=40, H=7, W=9),                      # two channel groups, the second ragged
    small(B=1, D=33, H=14, W=14),                    # VMamba-B's 14 x 14 map, 13 chunks
    small(B=1, D=8, H=33, W=31),                     # L = 1023: 64 chunks
    small(B=2, D=5, H=3, W=4),                       # L = 12: one chunk
    small(B=2, D=9, H=6, W=5, K=2, N=5),
    small(B=2, D=9, H=6, W=5, K=1, N=1),
    small("1d", B=3, D=20, W=197, K=2, N=16),        # Vim-S's 197 tokens
    small("1d", B=2, D=7, W=50, K=1, N=3),
    small("1d", B=1, D=33, W=1000, K=2, N=16),
]


@pytest.mark.parametrize("cfg", SHAPES, ids=lambda c: c.name)
@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16, wl.F16])
def test_backward_matches_oracle(cfg, dtype):
    cfg = cfg.with_(dtype=dtype)
    inp = wl.make_inputs(cfg, seed=2)
    dy = wl.make_cotangent(cfg, seed=2)
    assert_grads_close(gpu_backward(inp, dy), oracle_backward(inp, dy), cfg.name)


@pytest.mark.parametrize("cfg", SHAPES + [small(B=2, D=12, H=7, W=9, N=20),
                                          small(B=1, D=40, H=14, W=14, N=40),
                                          small(B=2, D=9, H=6, W=5, K=2, N=64),
                                          small("1d", B=3, D=20, W=197, K=2, N=33)],
                         ids=lambda c: c.name)
def test_backward_row_parameters_and_state_groups(cfg):
    """A_log and Dskip different in every row (k, d), and state counts above
    16 (groups of 16 states run one after the other)."""
    inp = _gpu.vary_params(wl.make_inputs(cfg, seed=13), seed=13)
    dy = wl.make_cotangent(cfg, seed=13)
    assert_grads_close(gpu_backward(inp, dy), oracle_backward(inp, dy), cfg.name + " varied")


@pytest.mark.parametrize("cfg", [small(B=8, D=1024, H=16, W=16, K=4, N=16),
                                 small(B=24, D=1024, H=6, W=8, K=4, N=16)],
                         ids=["ranges_of_6_chunks", "one_range_per_sequence"])
def test_backward_chunk_ranges(cfg):
    """Enough channels that a CTA walks several chunks (the adjoint carried
    from chunk to chunk inside the kernel, G from the carry only at the top
    of each range), and so many that one range covers a whole sequence (no
    local adjoints, no adjoint carry)."""
    inp = _gpu.vary_params(wl.make_inputs(cfg, seed=14), seed=14)
    dy = wl.make_cotangent(cfg, seed=14)
    assert_grads_close(gpu_backward(inp, dy), oracle_backward(inp, dy), cfg.name)


def test_backward_large_dt():
    """dt of order one (delta_bias = 0), where every term of the gradient,
    the decay terms included, carries weight."""
    cfg = small(B=2, D=24, H=10, W=12)
    inp = wl.make_inputs(cfg, seed=5)
    inp.delta_bias[:] = 0.0
    dy = wl.make_cotangent(cfg, seed=5)
    assert_grads_close(gpu_backward(inp, dy), oracle_backward(inp, dy), "large dt")


def test_backward_deterministic():
    cfg = small(B=2, D=70, H=12, W=20, dtype=wl.BF16)
    inp = wl.make_inputs(cfg, seed=3)
    dy = wl.make_cotangent(cfg, seed=3)
    t = _gpu.tensors(inp)
    a, b = gpu_backward(inp, dy, t), gpu_backward(inp, dy, t)
    for n in GRADS:
        assert np.array_equal(a[n], b[n]), n


def test_backward_deterministic_two_directions():
    # K = 2: both directions add their du into dx (atomic adds of two terms)
    cfg = small("1d", B=2, D=70, W=203, K=2, dtype=wl.BF16)
    inp = wl.make_inputs(cfg, seed=4)
    dy = wl.make_cotangent(cfg, seed=4)
    t = _gpu.tensors(inp)
    a, b = gpu_backward(inp, dy, t), gpu_backward(inp, dy, t)
    for n in GRADS:
        assert np.array_equal(a[n], b[n]), n


def test_zero_cotangent_gives_zero_gradients():
    cfg = small(B=2, D=12, H=9, W=9)
    inp = wl.make_inputs(cfg, seed=1)
    g = gpu_backward(inp, np.zeros((2, 12, 9, 9), np.float32))
    for n in GRADS:
        assert not np.any(g[n]), n


def test_empty_batch_zeroes_parameter_gradients():
    cfg = small(B=0, D=6, H=4, W=4)
    inp = wl.make_inputs(cfg, seed=0)
    t = _gpu.tensors(inp)
    g = binding.ss2d_backward(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"],
                              t["delta_bias"], torch.zeros((0, 6, 4, 4), device="cuda"))
    torch.cuda.synchronize()
    for n in ("dA_log", "dDskip", "ddelta_bias"):
        assert g[n].numel() > 0 and not torch.any(g[n]), n


def test_backward_rejects_host_pointers():
    inp = wl.make_inputs(small(B=1, D=4, H=4, W=4, N=4), seed=0)
    th = _gpu.tensors(inp, device=None)
    td = _gpu.tensors(inp)
    lib = binding.lib()
    gd = [torch.empty(s, device="cuda") for s in ((1, 4, 4, 4), (1, 4, 4, 16), (16, 4),
                                                  (1, 4, 4, 16), (1, 4, 4, 16), (16,), (16,))]
    names = ("x", "delta", "A_log", "Bs", "Cs", "Dskip", "delta_bias")
    dy = torch.zeros((1, 4, 4, 4))
    rc = lib.ss2d_backward(*[binding._ptr(th[n]) for n in names], binding._ptr(dy),
                           *[binding._ptr(g) for g in gd], 1, 4, 4, 4, 4, 4, 0, None)
    assert rc == -9
    rc = lib.ss2d_backward(*[binding._ptr(td[n]) for n in names], binding._ptr(dy),
                           *[binding._ptr(g) for g in gd], 1, 4, 4, 4, 4, 4, 0, None)
    assert rc == -9   # dy on the host, the rest on the device


# ---------------------------------------------------------------------------
# full-size workloads: batch element 0 against the oracle (every channel, so
# the channel sums of dBs, dCs are checked too), and the batch sums of the
# parameter gradients against the sum of per-element GPU calls
# ---------------------------------------------------------------------------
FULL = ["vmamba_t_stage1", "vmamba_b_stage3", "vim_s_bidir"]


@pytest.mark.parametrize("name", FULL)
def test_backward_full_size(name):
    inp = wl.make_inputs(name, seed=0)
    cfg = inp.cfg
    dy = wl.make_cotangent(cfg, seed=0)
    t = _gpu.tensors(inp)
    full = gpu_backward(inp, dy, t)
    sub = wl.batch_subproblem(inp, 0)
    ref0 = oracle_backward(sub, dy[:1])
    got0 = {n: (v[:1] if n in ("dx", "ddelta", "dBs", "dCs") else v) for n, v in full.items()}
    assert_grads_close(got0, ref0, name + " batch 0", names=("dx", "ddelta", "dBs", "dCs"))
    # parameter gradients: batch element 0 alone against the oracle, and the
    # full batch against the sum of per-element calls (fixed-order sums of
    # the same partials, so equal up to float32 rounding)
    one = gpu_backward(sub, np.ascontiguousarray(dy[:1]))
    assert_grads_close(one, ref0, name + " batch 0 alone")
    acc = {n: np.zeros_like(full[n]) for n in ("dA_log", "dDskip", "ddelta_bias")}
    for b in range(cfg.B):
        g = gpu_backward(wl.batch_subproblem(inp, b), np.ascontiguousarray(dy[b:b + 1]))
        for n in acc:
            acc[n] += g[n]
    assert_grads_close(full, acc, name + " batch sums", names=tuple(acc))


def test_backward_highres_sampled_channels():
    """256 x 256 (L = 65536): the input gradients of sampled channels against
    the oracle run on that channel alone (they depend on no other channel)."""
    inp = wl.make_inputs("highres_256", seed=0)
    dy = wl.make_cotangent(inp.cfg, seed=0)
    full = gpu_backward(inp, dy)
    for d in (0, 97, 191):
        sub = wl.channel_subproblem(inp, 0, d)
        ref = oracle_backward(sub, np.ascontiguousarray(dy[:1, d:d + 1]))
        got = {"dx": full["dx"][:1, d:d + 1], "ddelta": full["ddelta"][:1, :, d:d + 1]}
        assert_grads_close(got, ref, f"highres channel {d}", names=("dx", "ddelta"))

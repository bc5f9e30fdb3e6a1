"""ss2d_forward_noalloc: the forward call whose scratch is a fixed device
buffer of the library instead of the stream pool.

Host tests (no GPU): the entry point is exported, and a problem whose scratch
would not fit is refused with SS2D_ERR_SCRATCH before any CUDA call.
GPU tests: two calls in a row match ss2d_forward within the parity tolerance
(fp32 per element, bf16 relative L2) on chunked and unchunked shapes and on
K = 1, 2, 4; an oversize problem with real device buffers is refused and y is
left untouched; repeated calls leave the device's free memory unchanged.
The file is named to be collected last, and it also passes on its own in a
fresh process (the first call sets the buffer up)."""
import ctypes

import numpy as np
import pytest
import torch

import _gpu
from selective_scan_ss2d_b200 import binding, build
from selective_scan_ss2d_b200 import workloads as wl

SS2D_ERR_SCRATCH = -11


def scratch_bytes(B, D, H, W, N, K):
    """Scratch the call needs, as the header states it."""
    nc = binding.ss2d_plan(True, B, D, H, W, N, K)["num_chunks"]
    r = lambda v: (v + 255) // 256 * 256
    part = r(4 * B * K * D * H * W) if (K == 4 or (K == 2 and N > 16)) else 0
    states = r(64 * B * K * D * (nc - 1)) + r(4 * B * K * D * (nc - 1)) if nc > 1 else 0
    return part + states


# --------------------------------------------------------------------- host
@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def test_noalloc_exported(lib):
    assert hasattr(lib, "ss2d_forward_noalloc")
    assert binding.ss2d_status_string(SS2D_ERR_SCRATCH) != "unknown status"


def test_noalloc_refuses_oversize_before_cuda(lib):
    # B=8, D=256, 64x64, K=4: 128 MiB of scan-order rows alone
    B, D, H, W, N, K = 8, 256, 64, 64, 16, 4
    assert scratch_bytes(B, D, H, W, N, K) > binding.NOALLOC_SCRATCH_BYTES
    buf = (ctypes.c_float * 64)()
    a = ctypes.addressof(buf)
    p = ctypes.c_void_p((a + 15) // 16 * 16)
    rc = lib.ss2d_forward_noalloc(p, p, p, p, p, p, p, p, B, D, H, W, N, K, 1, None)
    assert rc == SS2D_ERR_SCRATCH
    assert b"scratch needed" in lib.ss2d_last_error()


def test_noalloc_shape_rules_match_forward(lib):
    p = ctypes.c_void_p(0)
    assert lib.ss2d_forward_noalloc(p, p, p, p, p, p, p, p, 1, 1, 2, 2, 4, 3, 0, None) == -4
    assert lib.ss2d_forward_noalloc(p, p, p, p, p, p, p, p, 1, 1, 2, 2, 65, 4, 0, None) == -5
    assert lib.ss2d_forward_noalloc(p, p, p, p, p, p, p, p, 1, 1, 2, 2, 4, 4, 7, None) == -3
    assert lib.ss2d_forward_noalloc(p, p, p, p, p, p, p, p, 0, 1, 2, 2, 4, 4, 0, None) == 0
    assert lib.ss2d_forward_noalloc(p, p, p, p, p, p, p, p, 1, 1, 2, 2, 4, 4, 0, None) == -1


# ---------------------------------------------------------------------- GPU
def cfg(B, D, H, W, K, N, dtype):
    return wl.Config(f"noalloc_{B}_{D}_{H}x{W}_{K}_{N}_{dtype}", "2d", B, D, H, W, K, N, dtype)


SHAPES = [
    cfg(1, 8, 8, 8, 4, 4, wl.F32),        # the tiny workload's shape
    cfg(2, 40, 7, 9, 4, 16, wl.F32),      # ragged L = 63, two channel tiles
    cfg(2, 64, 12, 20, 4, 16, wl.BF16),
    cfg(1, 32, 40, 40, 4, 16, wl.BF16),   # chunked: L = 1600, few sequences
    cfg(1, 24, 30, 33, 2, 16, wl.F32),    # K = 2, chunked
    cfg(1, 16, 36, 36, 1, 8, wl.F32),     # K = 1: chunk states only
    cfg(1, 24, 30, 33, 4, 40, wl.BF16),   # N = 40: three state groups, chunked
]


@pytest.mark.gpu
@pytest.mark.parametrize("c", SHAPES, ids=lambda c: c.name)
def test_noalloc_matches_forward_two_calls(c):
    assert scratch_bytes(c.B, c.D, c.H, c.W, c.N, c.K) <= binding.NOALLOC_SCRATCH_BYTES
    inp = wl.make_inputs(c, seed=11)
    t = _gpu.tensors(inp, "cuda")
    args = (t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"])
    ref = binding.ss2d_forward(*args)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy().astype(np.float64)
    for call in range(2):
        y = torch.full((c.B, c.D, c.H, c.W), float("nan"), dtype=torch.float32, device="cuda")
        binding.ss2d_forward_noalloc(*args, y)
        torch.cuda.synchronize()
        _gpu.assert_close(y.cpu().numpy().astype(np.float64), ref, c.dtype,
                          f"{c.name} call {call}")


@pytest.mark.gpu
def test_noalloc_refuses_oversize_on_device():
    # B=4, D=192, 96x96, K=4: about 108 MiB of scratch, real buffers of that shape
    c = cfg(4, 192, 96, 96, 4, 16, wl.BF16)
    assert scratch_bytes(c.B, c.D, c.H, c.W, c.N, c.K) > binding.NOALLOC_SCRATCH_BYTES
    L = c.H * c.W
    dev = "cuda"
    x = torch.zeros((c.B, c.D, c.H, c.W), dtype=torch.bfloat16, device=dev)
    delta = torch.zeros((c.B, c.K, c.D, L), dtype=torch.bfloat16, device=dev)
    Bs = torch.zeros((c.B, c.K, c.N, L), dtype=torch.bfloat16, device=dev)
    Cs = torch.zeros_like(Bs)
    A_log = torch.zeros((c.K * c.D, c.N), dtype=torch.float32, device=dev)
    Dskip = torch.ones(c.K * c.D, dtype=torch.float32, device=dev)
    bias = torch.zeros(c.K * c.D, dtype=torch.float32, device=dev)
    y = torch.full((c.B, c.D, c.H, c.W), 7.0, dtype=torch.float32, device=dev)
    with pytest.raises(binding.SS2DError) as ei:
        binding.ss2d_forward_noalloc(x, delta, A_log, Bs, Cs, Dskip, bias, y)
    assert ei.value.status == SS2D_ERR_SCRATCH
    torch.cuda.synchronize()
    assert bool(torch.all(y == 7.0))


@pytest.mark.gpu
def test_noalloc_leaves_free_memory_unchanged():
    c = cfg(1, 32, 40, 40, 4, 16, wl.BF16)
    inp = wl.make_inputs(c, seed=12)
    t = _gpu.tensors(inp, "cuda")
    args = (t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"])
    y = torch.empty((c.B, c.D, c.H, c.W), dtype=torch.float32, device="cuda")
    binding.ss2d_forward_noalloc(*args, y)          # first call: buffer address, kernels
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        binding.ss2d_forward_noalloc(*args, y)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0

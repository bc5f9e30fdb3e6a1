"""The C-ABI library on the host (no GPU needed): it loads, exports every
function include/ss2d.h declares, and rejects bad arguments with the
documented status codes before it touches CUDA."""
import ctypes
import os
import re

import pytest

from selective_scan_ss2d_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("ss2d_forward", "selective_scan_fwd", "ss2d_status_string"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_status_strings(lib):
    for st in range(0, -12, -1):
        s = binding.ss2d_status_string(st)
        assert s and s != "unknown status"
    assert binding.ss2d_status_string(-99) == "unknown status"
    # every forward and backward entry takes N in 1..64; only the timed call
    # is limited to one group of 16
    assert "1..64" in binding.ss2d_status_string(-5)
    assert "1..16 for ss2d_forward_timed" in binding.ss2d_status_string(-5)


def test_variant_table(lib):
    n = binding.ss2d_num_variants()
    assert n >= 4
    names = [binding.ss2d_variant_name(i) for i in range(n)]
    assert all(names) and len(set(names)) == n
    assert binding.ss2d_variant_name(n) == ""


@pytest.mark.parametrize("shape", [(1, 8, 8, 8, 4, 4), (8, 192, 56, 56, 16, 4),
                                   (64, 1024, 14, 14, 16, 4), (1, 192, 256, 256, 16, 4)])
def test_pick_variant_in_range(lib, shape):
    B, D, H, W, N, K = shape
    v = binding.ss2d_pick_variant(True, B, D, H, W, N, K)
    assert 0 <= v < binding.ss2d_num_variants()
    assert 0 <= binding.ss2d_pick_variant(False, 128, 768, 1, 197, 16, 2) < binding.ss2d_num_variants()


def _call(lib, ptr, B=1, D=1, H=2, W=2, N=4, K=4, dtype=0, variant=-1, two_d=True, nulls=()):
    args = [ptr] * 8
    for i in nulls:
        args[i] = None
    if two_d:
        return lib.ss2d_forward_ex(*args, B, D, H, W, N, K, dtype, None, variant)
    return lib.selective_scan_fwd_ex(*args, B, D, H * W, N, K, dtype, None, variant)


def test_argument_errors_are_reported_without_cuda(lib):
    buf = (ctypes.c_float * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    addr = ctypes.addressof(buf)
    aligned = ctypes.c_void_p(addr + (-addr) % 16)
    assert _call(lib, aligned, B=-1) == -2
    assert _call(lib, aligned, W=-3) == -2
    assert _call(lib, aligned, dtype=7) == -3
    assert _call(lib, aligned, K=3) == -4
    assert _call(lib, aligned, K=4, two_d=False) == -4
    assert _call(lib, aligned, N=0) == -5
    assert _call(lib, aligned, N=65) == -5
    assert _call(lib, aligned, variant=10_000) == -10
    assert _call(lib, aligned, nulls=(3,)) == -1
    assert _call(lib, aligned, nulls=(7,)) == -1
    misaligned = ctypes.c_void_p(aligned.value + 4)
    assert _call(lib, misaligned) == -6
    assert _call(lib, aligned, B=70000) == -2
    # empty problems are valid and do nothing (pointers are not read)
    assert _call(lib, aligned, B=0, nulls=range(8)) == 0
    assert _call(lib, aligned, H=0, nulls=range(8)) == 0
    assert _call(lib, aligned, D=0, K=2, two_d=False, nulls=range(8)) == 0
    assert p is not None


def test_binding_validates_tensors(lib):
    import torch
    x = torch.zeros(1, 2, 3, 3)
    delta = torch.zeros(1, 4, 2, 9)
    Bs = torch.zeros(1, 4, 4, 9)
    A_log = torch.zeros(8, 4)
    Dk = torch.zeros(8)
    with pytest.raises(ValueError):
        binding.ss2d_forward(x, delta, A_log, Bs, Bs[:, :, :3], Dk, Dk)
    with pytest.raises(TypeError):
        binding.ss2d_forward(x.double(), delta, A_log, Bs, Bs, Dk, Dk)
    with pytest.raises(TypeError):
        binding.ss2d_forward(x, delta.bfloat16(), A_log, Bs, Bs, Dk, Dk)
    with pytest.raises(ValueError):
        binding.ss2d_forward(x, delta, A_log, Bs.transpose(2, 3).contiguous().transpose(2, 3),
                             Bs, Dk, Dk)


def test_plans_for_the_workloads(lib):
    from selective_scan_ss2d_b200 import workloads as wl
    for name, cfg in wl.CONFIGS.items():
        pl = binding.ss2d_plan(cfg.kind == "2d", cfg.B, cfg.D, cfg.H, cfg.W, cfg.N, cfg.K)
        assert pl["chunk_len"] % 16 == 0
        assert pl["num_chunks"] == -(-cfg.L // pl["chunk_len"])
        nc = pl["num_chunks"]
        # state pass, carry (not needed with two chunks), output pass; merge
        # (K = 2 with at most 16 states merges in the output pass)
        merge = 1 if cfg.K == 4 or (cfg.K == 2 and cfg.N > 16) else 0
        want = (3 if nc > 2 else 2 if nc > 1 else 1) + merge
        assert pl["launches"] == want
    # long sequences with few channels are chunked, short ones are not
    t = wl.CONFIGS["vmamba_t_stage1"]
    assert binding.ss2d_plan(True, t.B, t.D, t.H, t.W, t.N, t.K)["num_chunks"] > 1
    b = wl.CONFIGS["vmamba_b_stage3"]
    assert binding.ss2d_plan(True, b.B, b.D, b.H, b.W, b.N, b.K)["num_chunks"] == 1


def _bwd_call(lib, ptr, B=1, D=1, H=2, W=2, N=4, K=4, dtype=0, two_d=True, nulls=()):
    args = [ptr] * 15   # seven inputs, dy, seven gradients
    for i in nulls:
        args[i] = None
    if two_d:
        return lib.ss2d_backward(*args, B, D, H, W, N, K, dtype, None)
    return lib.selective_scan_bwd(*args, B, D, H * W, N, K, dtype, None)


def test_backward_argument_errors_are_reported_without_cuda(lib):
    buf = (ctypes.c_float * 64)()
    addr = ctypes.addressof(buf)
    aligned = ctypes.c_void_p(addr + (-addr) % 16)
    assert _bwd_call(lib, aligned, B=-1) == -2
    assert _bwd_call(lib, aligned, dtype=9) == -3
    assert _bwd_call(lib, aligned, K=3) == -4
    assert _bwd_call(lib, aligned, K=4, two_d=False) == -4
    assert _bwd_call(lib, aligned, N=65) == -5
    for i in (0, 7, 8, 14):   # x, dy, dx, ddelta_bias
        assert _bwd_call(lib, aligned, nulls=(i,)) == -1
    assert _bwd_call(lib, ctypes.c_void_p(aligned.value + 4)) == -6


def test_backward_binding_validates_tensors(lib):
    import torch
    x = torch.zeros(1, 2, 3, 3)
    delta = torch.zeros(1, 4, 2, 9)
    Bs = torch.zeros(1, 4, 4, 9)
    A_log = torch.zeros(8, 4)
    Dk = torch.zeros(8)
    with pytest.raises(ValueError, match="dy"):
        binding.ss2d_backward(x, delta, A_log, Bs, Bs, Dk, Dk, torch.zeros(1, 2, 3, 4))
    with pytest.raises(ValueError, match="dy"):
        binding.ss2d_backward(x, delta, A_log, Bs, Bs, Dk, Dk, x.double())
    with pytest.raises(ValueError, match="device tensors only"):
        binding.ss2d_backward(x, delta, A_log, Bs, Bs, Dk, Dk, x.clone())
    with pytest.raises(ValueError, match="inconsistent"):
        binding.selective_scan_bwd(x[:, :, 0], delta, A_log, Bs, Bs, Dk, Dk, x[:, :, 0].clone())


def test_final_state_argument_errors_are_reported_without_cuda(lib):
    buf = (ctypes.c_float * 64)()
    addr = ctypes.addressof(buf)
    p = ctypes.c_void_p(addr + (-addr) % 16)
    args = [p] * 8
    # h_last missing: SS2D_ERR_NULL before anything else
    assert lib.ss2d_forward_final_state(*args, None, 1, 1, 2, 2, 4, 4, 0, None, -1) == -1
    assert lib.selective_scan_fwd_final_state(*args, None, 1, 1, 4, 4, 2, 0, None, -1) == -1
    # then the forward's own rules
    assert lib.ss2d_forward_final_state(*args, p, 1, 1, 2, 2, 65, 4, 0, None, -1) == -5
    assert lib.ss2d_forward_final_state(*args, p, 1, 1, 2, 2, 4, 3, 0, None, -1) == -4
    assert lib.selective_scan_fwd_final_state(*args, p, 1, 1, 4, 4, 4, 0, None, -1) == -4
    assert lib.ss2d_forward_final_state(*args, p, 1, 1, 2, 2, 4, 4, 0, None, 10_000) == -10


def test_plan_counts_launches_per_state_group(lib):
    one = binding.ss2d_plan(True, 8, 192, 56, 56, 16, 4)
    three = binding.ss2d_plan(True, 8, 192, 56, 56, 40, 4)
    assert one["num_chunks"] == three["num_chunks"] > 1
    # three groups of states: three (state pass, carry, output pass), one merge
    assert one["launches"] == 3 + 1 and three["launches"] == 3 * 3 + 1
    # K = 2: merged in the output pass with one state group, a merge launch with more
    assert binding.ss2d_plan(False, 128, 768, 1, 197, 16, 2)["launches"] == 1
    assert binding.ss2d_plan(False, 128, 768, 1, 197, 24, 2)["launches"] == 2 + 1


def test_final_state_binding_validates_tensors(lib):
    import torch
    x = torch.zeros(1, 2, 3, 3)
    delta = torch.zeros(1, 4, 2, 9)
    Bs = torch.zeros(1, 4, 4, 9)
    A_log = torch.zeros(8, 4)
    Dk = torch.zeros(8)
    with pytest.raises(ValueError, match="device tensors only"):
        binding.forward_final_state(x, delta, A_log, Bs, Bs, Dk, Dk)
    with pytest.raises(ValueError, match="inconsistent"):
        binding.forward_final_state(x, delta[:, :2], A_log, Bs, Bs, Dk, Dk)
    u = torch.zeros(1, 2, 9)
    with pytest.raises(ValueError, match="inconsistent"):
        binding.forward_final_state(u, delta, A_log, Bs, Bs[:, :, :3], Dk, Dk)
    with pytest.raises(TypeError):
        binding.selective_scan_bwd(u.double(), delta, A_log, Bs, Bs, Dk, Dk, u.clone())

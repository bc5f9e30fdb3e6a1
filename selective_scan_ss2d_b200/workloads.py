"""Seeded synthetic workloads for the SS2D forward path.

This module draws inputs and nothing else: it holds none of the method's
arithmetic.  The same arrays feed the CUDA library and the float64 oracle, so
both see identical values (bf16 and fp16 inputs are rounded here once, and
the oracle reads those rounded values back as float64).

Shapes follow the models the pages describe: the VMamba hierarchy ("Vision
Mamba" tutorial, section "VMamba Hierarchical Architecture": 4x4 patches,
stage widths 96/192/384/768, so a 224x224 image gives a 56x56 stage-1 map and
a 14x14 stage-3 map), an inner width of twice the model width, state size 16
(SelectiveSSM's default), and Vim-S (16x16 patches of a 224x224 image plus one
class token: 197 tokens; "Vision Mamba ..." summary, section 4.2).

Recipe (seeded NumPy PCG64, one generator per workload, draws in this order):
x (or u), delta, Bs, Cs ~ N(0, 1) in float32; then dt = exp(U[ln 1e-3, ln 1e-1])
per row k*D+d; delta_bias = softplus^-1(dt) = ln(expm1(dt)); A_log[kd, n] =
ln(n + 1) (the tutorial's initialisation of A); Dskip = 1.  For bf16
workloads x, delta, Bs and Cs are rounded to bfloat16, for f16 workloads to
IEEE float16 (both round to nearest, ties to even).  Parameters stay float32.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

F32 = "f32"
BF16 = "bf16"
F16 = "f16"   # IEEE binary16 storage (float16 arrays)


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    kind: str          # "2d" (ss2d_forward) or "1d" (selective_scan_fwd)
    B: int
    D: int
    H: int             # 1 for the 1D kind
    W: int             # L for the 1D kind
    K: int
    N: int
    dtype: str
    description: str = ""

    @property
    def L(self) -> int:
        return self.H * self.W

    @property
    def updates(self) -> int:
        """State updates per forward pass: B*K*D*L*N."""
        return self.B * self.K * self.D * self.L * self.N

    @property
    def in_bytes_per_elem(self) -> int:
        return 4 if self.dtype == F32 else 2

    @property
    def algorithmic_bytes(self) -> int:
        """x (or u), delta, Bs and Cs read once; y (float32) written once.
        The parameter vectors (K*D*(N+2) float32) are counted too."""
        e = self.in_bytes_per_elem
        x = self.B * self.D * self.L * e
        delta = self.B * self.K * self.D * self.L * e
        bc = 2 * self.B * self.K * self.N * self.L * e
        y = self.B * self.D * self.L * 4
        params = self.K * self.D * (self.N + 2) * 4
        return x + delta + bc + y + params

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny_fp32": Config("tiny_fp32", "2d", 1, 8, 8, 8, 4, 4, F32,
                        "Tiny SS2D, fp32: B=1, D=8, H=W=8 (L=64), K=4, N=4"),
    "vmamba_t_stage1": Config("vmamba_t_stage1", "2d", 8, 192, 56, 56, 4, 16, BF16,
                              "VMamba-T stage-1 SS2D: B=8, D=192, H=W=56 (L=3136), K=4, N=16"),
    "vmamba_b_stage3": Config("vmamba_b_stage3", "2d", 64, 1024, 14, 14, 4, 16, BF16,
                              "VMamba-B stage-3 SS2D: B=64, D=1024, H=W=14 (L=196), K=4, N=16"),
    "highres_256": Config("highres_256", "2d", 1, 192, 256, 256, 4, 16, BF16,
                          "High-resolution SS2D: B=1, D=192, H=W=256 (L=65536), K=4, N=16"),
    "vim_s_bidir": Config("vim_s_bidir", "1d", 128, 768, 1, 197, 2, 16, BF16,
                          "Vim-S bidirectional 1D scan: B=128, D=768, L=197, K=2, N=16"),
}
CONFIG_ORDER = ["tiny_fp32", "vmamba_t_stage1", "vmamba_b_stage3", "highres_256",
                "vim_s_bidir"]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16, nearest with ties to even; returns
    the 16-bit patterns.  (Finite inputs only.)"""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Inputs:
    """One workload's arrays in storage form: float32, uint16 bfloat16
    patterns (bf16 workloads) or float16 (f16 workloads) for the four streamed
    inputs."""
    cfg: Config
    x: np.ndarray          # (B,D,H,W) or (B,D,L)
    delta: np.ndarray      # (B,K,D,L)
    Bs: np.ndarray         # (B,K,N,L)
    Cs: np.ndarray         # (B,K,N,L)
    A_log: np.ndarray      # (K*D,N) float32
    Dskip: np.ndarray      # (K*D,) float32
    delta_bias: np.ndarray  # (K*D,) float32

    STREAMED = ("x", "delta", "Bs", "Cs")
    PARAMS = ("A_log", "Dskip", "delta_bias")

    def as_f64(self) -> dict:
        """The exact values the GPU sees, widened to float64."""
        out = {}
        for name in self.STREAMED:
            a = getattr(self, name)
            if self.cfg.dtype == BF16:
                a = bf16_bits_to_f32(a)
            out[name] = a.astype(np.float64)
        for name in self.PARAMS:
            out[name] = getattr(self, name).astype(np.float64)
        return out

    def arrays(self) -> dict:
        return {n: getattr(self, n) for n in self.STREAMED + self.PARAMS}


def _normal(rng, shape, dtype):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype == BF16:
        return f32_to_bf16_bits(a).reshape(shape)
    if dtype == F16:
        return a.astype(np.float16)   # IEEE round to nearest, ties to even
    return a


def make_inputs(cfg: Config | str, seed: int = 0) -> Inputs:
    """Draw one workload (see the module docstring for the recipe)."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    rng = np.random.default_rng(seed)
    B, D, K, N, L = cfg.B, cfg.D, cfg.K, cfg.N, cfg.L
    xshape = (B, D, cfg.H, cfg.W) if cfg.kind == "2d" else (B, D, L)
    x = _normal(rng, xshape, cfg.dtype)
    delta = _normal(rng, (B, K, D, L), cfg.dtype)
    Bs = _normal(rng, (B, K, N, L), cfg.dtype)
    Cs = _normal(rng, (B, K, N, L), cfg.dtype)
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=K * D))
    delta_bias = np.log(np.expm1(dt)).astype(np.float32)
    A_log = np.repeat(np.log(np.arange(1, N + 1, dtype=np.float64))[None, :],
                      K * D, axis=0).astype(np.float32)
    Dskip = np.ones(K * D, dtype=np.float32)
    return Inputs(cfg, x, delta, Bs, Cs, A_log, Dskip, delta_bias)


def make_gate(cfg: Config | str, seed: int = 0) -> np.ndarray:
    """The gate input z of a gated call: N(0, 1) in the layout of x, in the
    workload's storage dtype (a stream of its own, so the other inputs of the
    same seed are unchanged)."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    rng = np.random.default_rng([seed, 0x6a7e])
    xshape = (cfg.B, cfg.D, cfg.H, cfg.W) if cfg.kind == "2d" else (cfg.B, cfg.D, cfg.L)
    return _normal(rng, xshape, cfg.dtype)


def make_cotangent(cfg: Config | str, seed: int = 0) -> np.ndarray:
    """The cotangent dy of a backward call: N(0, 1) float32 in the layout of
    y (a stream of its own, so the other inputs of the same seed are
    unchanged)."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    rng = np.random.default_rng([seed, 0xd1])
    xshape = (cfg.B, cfg.D, cfg.H, cfg.W) if cfg.kind == "2d" else (cfg.B, cfg.D, cfg.L)
    return rng.standard_normal(size=xshape, dtype=np.float32)


def gate_as_f64(z: np.ndarray, cfg: Config) -> np.ndarray:
    """The exact values a gated call sees, widened to float64."""
    return (bf16_bits_to_f32(z) if cfg.dtype == BF16 else z).astype(np.float64)


def channel_subproblem(inp: Inputs, b: int, d: int) -> Inputs:
    """The inputs that one output channel (b, d) depends on, as a B=1, D=1
    workload of its own (pure slicing; used to check sampled channels of a
    full-size run against the oracle)."""
    cfg = inp.cfg
    K, D = cfg.K, cfg.D
    rows = [k * D + d for k in range(K)]
    sub = cfg.with_(name=f"{cfg.name}[b={b},d={d}]", B=1, D=1)
    return Inputs(sub,
                  np.ascontiguousarray(inp.x[b:b + 1, d:d + 1]),
                  np.ascontiguousarray(inp.delta[b:b + 1, :, d:d + 1]),
                  np.ascontiguousarray(inp.Bs[b:b + 1]),
                  np.ascontiguousarray(inp.Cs[b:b + 1]),
                  np.ascontiguousarray(inp.A_log[rows]),
                  np.ascontiguousarray(inp.Dskip[rows]),
                  np.ascontiguousarray(inp.delta_bias[rows]))


def batch_subproblem(inp: Inputs, b: int) -> Inputs:
    """Batch element b of a workload as a B=1 workload of its own (pure
    slicing; every channel kept)."""
    sub = inp.cfg.with_(name=f"{inp.cfg.name}[b={b}]", B=1)
    return Inputs(sub, *[np.ascontiguousarray(getattr(inp, n)[b:b + 1]) for n in Inputs.STREAMED],
                  inp.A_log, inp.Dskip, inp.delta_bias)


# ---------------------------------------------------------------------------
# the fused front's inputs
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class FrontConfig:
    name: str
    B: int
    L: int
    D: int
    N: int
    K: int
    dtype: str
    description: str = ""

    @property
    def updates(self) -> int:
        return self.B * self.K * self.D * self.L * self.N

    def with_(self, **kw) -> "FrontConfig":
        return dataclasses.replace(self, **kw)


FRONT_CONFIGS = {
    "vim_s_front": FrontConfig(
        "vim_s_front", 128, 197, 768, 16, 2, BF16,
        "Vim-S bidirectional block, front + scan: B=128, L=197 tokens, D=768, K=2, N=16"),
}


@dataclasses.dataclass
class FrontInputs:
    """One front workload: x (B, L, D) in storage form (float32, uint16
    bfloat16 patterns or float16), the float32 weights of every direction and
    the scan parameters."""
    cfg: FrontConfig
    x: np.ndarray
    conv_w: np.ndarray      # (K, D, 4)
    conv_b: np.ndarray      # (K, D)
    W_x: np.ndarray         # (K, 1 + 2N, D)
    w_dt: np.ndarray        # (K, D)
    A_log: np.ndarray       # (K*D, N)
    Dskip: np.ndarray       # (K*D,)
    delta_bias: np.ndarray  # (K*D,)

    WEIGHTS = ("conv_w", "conv_b", "W_x", "w_dt", "A_log", "Dskip", "delta_bias")

    def x_f64(self) -> np.ndarray:
        a = bf16_bits_to_f32(self.x) if self.cfg.dtype == BF16 else self.x
        return a.astype(np.float64)


def make_front_inputs(cfg: FrontConfig | str, seed: int = 0) -> FrontInputs:
    """Seeded front inputs (PCG64, draws in this order): x ~ N(0, 1), conv
    taps ~ N(0, 1/2), conv bias ~ N(0, 0.1^2), W_x ~ N(0, 1/D) (unit-scale
    projections), w_dt ~ U(0.5, 1.5), then dt log-uniform in [1e-3, 1e-1] per
    row k*D+d with delta_bias = ln(expm1(dt)); A_log = ln(n + 1), Dskip = 1 as
    in the forward's recipe.  x is rounded to the storage dtype."""
    if isinstance(cfg, str):
        cfg = FRONT_CONFIGS[cfg]
    rng = np.random.default_rng(seed)
    B, L, D, N, K = cfg.B, cfg.L, cfg.D, cfg.N, cfg.K
    x = _normal(rng, (B, L, D), cfg.dtype)
    conv_w = (rng.standard_normal((K, D, 4)) * math.sqrt(0.5)).astype(np.float32)
    conv_b = (rng.standard_normal((K, D)) * 0.1).astype(np.float32)
    W_x = (rng.standard_normal((K, 1 + 2 * N, D)) / math.sqrt(D)).astype(np.float32)
    w_dt = rng.uniform(0.5, 1.5, (K, D)).astype(np.float32)
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=K * D))
    delta_bias = np.log(np.expm1(dt)).astype(np.float32)
    A_log = np.repeat(np.log(np.arange(1, N + 1, dtype=np.float64))[None, :],
                      K * D, axis=0).astype(np.float32)
    Dskip = np.ones(K * D, dtype=np.float32)
    return FrontInputs(cfg, x, conv_w, conv_b, W_x, w_dt, A_log, Dskip, delta_bias)

#!/usr/bin/env python
"""Throughput of the SS2D forward path on B200: state updates per second
(B*K*D*L*N / s) for one workload, plus its fraction of the HBM and exp-unit
rooflines.

A step is one full forward pass (cross_scan -> selective scan -> cross_merge)
over one batch of the workload, through the library's C ABI.  Inputs are
seeded synthetic arrays already resident in HBM; the L2 cache is flushed
(a write larger than L2) before every timed step, outside the step's events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
  python bench.py --impl reference ...   # the float64 CPU oracle, rank 0
  python bench.py --report               # one line per workload (not the
                                         # contract line; for the notes)
  python bench.py --backward [--config NAME]   # the gradient pass instead
  python bench.py --gate                 # the gated entry point (y * SiLU(z))
  python bench.py --front                # the fused front + scan of the Vim-S block
  python bench.py --dtype f16 --n-states 8     # another input dtype or N

At one GPU the default line also carries `per_config`: every other workload
of the set (tiny fp32, VMamba-B stage 3, the 256x256 map, Vim-S) timed the
same way with fewer steps, with its rooflines and a short oracle sample.

Multi-GPU (torchrun): the path has no exchange step, so every rank runs an
independent replica of the workload (weak scaling, no collective on the data
path); the barrier and the max-over-ranks time use NCCL.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("SS2D state updates/s (B·K·D·L·N) and % of HBM roofline, "
          "VMamba-T stage 1")
DEFAULT_CONFIG = "vmamba_t_stage1"
MUFU_EX2_PER_CLK_PER_SM = 16       # exp2 results per clock per SM (MUFU)
NUM_SMS = 148
FALLBACK_HBM_GBS = 6650.0
FALLBACK_SM_MAX_MHZ = 1965.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM bytes (read + write) per launch of the dominant kernel, from ncu
# captures of the output pass, keyed by workload; each entry carries
# the input dtype, the state count and the hash of the kernel sources it was
# taken from, and is reported only for that configuration while the sources
# are unchanged.
NCU_TRAFFIC = {
    # ncu captures of the output pass (L2 flushed before the kernel by ncu):
    # dram read 65407744 + write 25779200
    "vmamba_t_stage1": {"bytes": 91186944, "dtype": "bf16", "N": 16, "src": "2a5841823ef7a483"},
    # dram read 141930496 + write 161160704
    "vmamba_b_stage3": {"bytes": 303091200, "dtype": "bf16", "N": 16, "src": "2a5841823ef7a483"},
    # dram read 184888320 + write 156569344
    "highres_256": {"bytes": 341457664, "dtype": "bf16", "N": 16, "src": "2a5841823ef7a483"},
    # dram read 197712896 + write 38131456 (both directions add into y in L2)
    "vim_s_bidir": {"bytes": 235844352, "dtype": "bf16", "N": 16, "src": "2a5841823ef7a483"},
}

# the files that define the output pass (chunk_scan_kernel), its variant
# choice and its launch: the kernel the traffic figures above were taken from
FORWARD_KERNEL_SOURCES = ("ss2d_kernels.cuh", "ss2d_launch.cu", "ss2d_launch.h", "ss2d_params.h",
                          "ss2d_scan_bf16.cu", "ss2d_scan_f16.cu", "ss2d_scan_f32.cu",
                          "ss2d_scan_launch.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_scan_ss2d_b200", "csrc")
    for fn in FORWARD_KERNEL_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        bf16 = d.get("bf16_tflops")
        return {"hbm_gbs": float(d["hbm_gbs"]),
                "sm_max_mhz": float(d.get("sm_max_mhz", FALLBACK_SM_MAX_MHZ)),
                "bf16_tflops": float(bf16) if bf16 else FALLBACK_BF16_TFLOPS,
                "bf16_source": "measured (bf16_tflops, burst)" if bf16 else "fallback",
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": FALLBACK_SM_MAX_MHZ,
            "bf16_tflops": FALLBACK_BF16_TFLOPS, "bf16_source": "fallback", "source": "fallback"}


# ---------------------------------------------------------------------------
# ranks: one process per GPU, no collective on the data path
# ---------------------------------------------------------------------------
def init_distributed(world: int, local_rank: int, backend: str = "nccl") -> None:
    """Join the job's process group (torchrun's env://) when world > 1."""
    if world <= 1:
        return
    import datetime
    import torch
    import torch.distributed as dist
    if backend == "nccl":
        torch.cuda.set_device(local_rank)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, device) -> float:
    """The maximum of x over all ranks (x itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: float, steps: int, world: int, max_total_ms: float) -> float:
    """Units per second of the whole job: every rank's units over the
    slowest rank's time."""
    return units_per_rank_step * steps * world / (max_total_ms / 1e3)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def _query_once(self):
        try:
            r = subprocess.run(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                "--format=csv,noheader,nounits"], capture_output=True,
                               text=True, timeout=10)
            return [ln for ln in r.stdout.splitlines() if ln.strip()]
        except Exception:
            return []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.lines.append(ln.strip())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)
        if not self.lines:
            self.lines = self._query_once()
        return self.summary()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def build_arrays(cfg, seed, device, pin=False):
    import numpy as np
    import torch
    from selective_scan_ss2d_b200 import workloads as wl
    inp = wl.make_inputs(cfg, seed=seed)
    out = {}
    for name in wl.Inputs.STREAMED + wl.Inputs.PARAMS:
        a = getattr(inp, name)
        t = (torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
             if a.dtype == np.uint16 else torch.from_numpy(np.ascontiguousarray(a)))
        if device is None:
            out[name] = t.pin_memory() if pin else t
        else:
            out[name] = t.to(device)
    return inp, out


def cpu_baseline_parallel(cfg, target_s: float, threads: int):
    """Time the float64 oracle, as it stands, on a bounded sample of the
    workload: whole output channels (all K directions over the full L), first
    the channels of batch element 0, then whole batch elements, grown until
    one call takes about target_s seconds.  The oracle's OpenMP loop spreads
    the channels over `threads` host cores.  Returns (updates/s, description,
    seconds)."""
    import oracle
    from selective_scan_ss2d_b200 import workloads as wl
    inp = wl.make_inputs(cfg, seed=0)
    fn = oracle.ss2d_forward if cfg.kind == "2d" else oracle.selective_scan_fwd

    def run(nb, nd):
        sub = slice_sample(inp, nb, nd)
        ff = sub.as_f64()
        t0 = time.perf_counter()
        fn(ff["x"], ff["delta"], ff["A_log"], ff["Bs"], ff["Cs"], ff["Dskip"], ff["delta_bias"],
           K=cfg.K, threads=threads)
        return time.perf_counter() - t0, sub.cfg.updates

    nb, nd = 1, min(cfg.D, max(threads, 1))
    dt, upd = run(nb, nd)
    while dt < target_s and (nd < cfg.D or nb < cfg.B):
        grow = max(2.0, target_s / max(dt, 1e-3))
        if nd < cfg.D:
            nd = min(cfg.D, int(nd * grow))
        else:
            nb = min(cfg.B, max(nb + 1, int(nb * grow)))
        dt, upd = run(nb, nd)
    desc = (f"batch elements 0..{nb - 1}, channels 0..{nd - 1} of {cfg.D}, all {cfg.K} "
            f"directions over the full L={cfg.L}: {upd} updates in {dt:.1f} s")
    return upd / dt, desc, dt


def slice_sample(inp, nb, nd):
    """Batch elements 0..nb-1, channels 0..nd-1 of a workload (pure slicing)."""
    import numpy as np
    from selective_scan_ss2d_b200 import workloads as wl
    cfg = inp.cfg
    K, D = cfg.K, cfg.D
    rows = [k * D + d for k in range(K) for d in range(nd)]
    sub = cfg.with_(name=f"{cfg.name}[b<{nb},d<{nd}]", B=nb, D=nd)
    return wl.Inputs(sub, np.ascontiguousarray(inp.x[:nb, :nd]),
                     np.ascontiguousarray(inp.delta[:nb, :, :nd]),
                     np.ascontiguousarray(inp.Bs[:nb]), np.ascontiguousarray(inp.Cs[:nb]),
                     np.ascontiguousarray(inp.A_log[rows]),
                     np.ascontiguousarray(inp.Dskip[rows]),
                     np.ascontiguousarray(inp.delta_bias[rows]))


def workload_config(name, dtype=None, n_states=None):
    """The named workload, with its streamed inputs' storage dtype (f32, bf16
    or f16) and its state count N replaced when given."""
    from selective_scan_ss2d_b200 import workloads as wl
    cfg = wl.CONFIGS[name]
    if dtype:
        cfg = cfg.with_(dtype=dtype)
    if n_states:
        cfg = cfg.with_(N=int(n_states))
    return cfg


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from selective_scan_ss2d_b200 import binding
    from selective_scan_ss2d_b200 import workloads as wl

    cfg = workload_config(args.config, args.dtype, args.n_states)
    dev = torch.device(f"cuda:{local_rank}")
    torch.cuda.set_device(dev)
    binding.lib()
    inp, t = build_arrays(cfg, seed=rank, device=dev)
    fn = binding.ss2d_forward if cfg.kind == "2d" else binding.selective_scan_fwd
    y = torch.empty(inp.x.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024) or 126 * 1024 * 1024
    flush = torch.empty(int(2 * l2) // 4, dtype=torch.float32, device=dev)

    gate = getattr(args, "gate", False)
    label = f"ss2d forward{' gated' if gate else ''} {cfg.name}"
    if gate:
        # the SiLU output gate: a seeded z in x's layout, the gated entry point
        # (the library's own variant choice)
        import numpy as np
        zr = wl.make_gate(cfg, seed=rank)
        zt = (torch.from_numpy(zr.view(np.int16)).view(torch.bfloat16) if zr.dtype == np.uint16
              else torch.from_numpy(zr)).to(dev)
        fn_g = binding.ss2d_forward_gated if cfg.kind == "2d" else binding.selective_scan_fwd_gated

    def step():
        if gate:
            fn_g(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"],
                 zt, y)
        else:
            fn(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"], y,
               variant=args.variant)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()

    gpu_id = str(getattr(props, "uuid", local_rank))
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) >= 32:
        gpu_id = "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.2)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push(f"{label} timed steps")   # marks the region for a trace
    for i in range(args.steps):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), dev)
    value = whole_job_rate(cfg.updates, args.steps, world, total_ms)

    # per-launch device times of the same calls (same inputs, same flushes),
    # CUDA events recorded by the library on this stream around each launch
    two_d = cfg.kind == "2d"
    per = []
    torch.cuda.nvtx.range_push(f"{label} per-launch timing")
    for i in range(args.steps):
        flush.fill_(float(i))
        per.append(binding.ss2d_forward_timed(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"],
                                              t["Dskip"], t["delta_bias"], y, two_d=two_d,
                                              stream=stream.cuda_stream, variant=args.variant))
    torch.cuda.nvtx.range_pop()
    names = ["chunk_state_pass", "carry", "scan_pass", "cross_merge"]
    launch_ms = {}
    for j, nm in enumerate(names):
        vals = [r[j] for r in per if r[j] >= 0]
        if vals:
            launch_ms[nm] = statistics.mean(vals)
    scan_ms = launch_ms["scan_pass"]

    result = {"rank_value": value}
    if rank == 0:
        peaks = measured_peaks()
        alg_bytes = cfg.algorithmic_bytes
        achieved_gbs = alg_bytes / (scan_ms / 1e3) / 1e9
        exps = cfg.updates + cfg.B * cfg.K * cfg.D * cfg.L
        mufu_peak = NUM_SMS * MUFU_EX2_PER_CLK_PER_SM * peaks["sm_max_mhz"] * 1e6 / 1e9
        achieved_gexp = exps / (scan_ms / 1e3) / 1e9
        src_hash = kernel_source_hash()
        tr = NCU_TRAFFIC.get(cfg.name)
        traffic = (tr["bytes"] if tr and tr.get("src") == src_hash and tr["dtype"] == cfg.dtype
                   and tr["N"] == cfg.N else None)
        variant = args.variant if args.variant >= 0 else binding.ss2d_pick_variant(
            two_d, cfg.B, cfg.D, cfg.H, cfg.W, cfg.N, cfg.K)
        plan = binding.ss2d_plan(two_d, cfg.B, cfg.D, cfg.H, cfg.W, cfg.N, cfg.K, variant)
        step_bytes = alg_bytes
        step_s = total_ms / args.steps / 1e3
        result["line"] = {
            "metric": METRIC,
            "value": value,
            "unit": "updates/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic (seeded N(0,1) inputs, rounded to the workload's bf16 or f16 storage)",
            "config": {"workload": cfg.name, "B": cfg.B, "D": cfg.D, "H": cfg.H, "W": cfg.W,
                       "L": cfg.L, "K": cfg.K, "N": cfg.N, "input_dtype": cfg.dtype,
                       "state_dtype": "f32", "updates_per_step": cfg.updates,
                       "algorithmic_bytes_per_step": step_bytes,
                       "kernel_variant": binding.ss2d_variant_name(variant),
                       "output_gate": "SiLU(z), gated entry point" if gate else None,
                       "l2": "flushed before every timed step (2x L2 write, outside events)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "alu", "achieved": achieved_gexp, "peak": mufu_peak,
                         "unit": "Gexp2/s", "frac": achieved_gexp / mufu_peak,
                         "traffic": traffic,
                         "kernel": "chunk_scan_kernel, output pass (every update of the step)",
                         "kernel_ms": scan_ms,
                         "peak_source": (f"MUFU exp2: {MUFU_EX2_PER_CLK_PER_SM}/clk/SM x "
                                         f"{NUM_SMS} SMs x {peaks['sm_max_mhz']:.0f} MHz "
                                         f"(sm_max_mhz, {peaks['source']})"),
                         "work": "1 exp2 per state update + 1 per (b,k,d,l) for softplus",
                         "step": {"achieved": exps / step_s / 1e9,
                                  "frac": exps / step_s / 1e9 / mufu_peak}},
            "roofline_hbm": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
                             "kernel_ms": scan_ms,
                             "peak_source": f"{peaks['source']} (hbm_gbs)",
                             "step": {"achieved": alg_bytes / step_s / 1e9,
                                      "frac": alg_bytes / step_s / 1e9 / peaks["hbm_gbs"]}},
            "launch_ms": launch_ms,
            "plan": plan,
            "gpu_launches": args.steps * plan["launches"],
        }
        result["clocks"] = clocks
    return result


def run_per_config(args, rank, world, local_rank):
    """The other workloads of the benchmark set, each timed like the
    headline (inputs resident, L2 flushed before every timed step, CUDA
    events) with fewer steps, and the float64 oracle on a bounded sample of
    each (about args.per_config_cpu_seconds of host time).  Returns
    {workload: summary} on rank 0."""
    from selective_scan_ss2d_b200 import workloads as wl
    out = {}
    for name in wl.CONFIG_ORDER:
        if name == args.config:
            continue
        a = argparse.Namespace(**vars(args))
        a.config = name
        a.steps = max(3, min(args.steps, args.per_config_steps))
        a.dtype = None
        a.n_states = None
        a.gate = False
        r = run_ours(a, rank, world, local_rank)
        if rank != 0:
            continue
        ln = r["line"]
        rf, rh = ln["roofline"], ln["roofline_hbm"]
        summary = {
            "config": ln["config"],
            "ms_per_step": ln["ms_per_step"],
            "value": ln["value"],
            "unit": ln["unit"],
            "steps": a.steps,
            "roofline": {"bound": rf["bound"], "unit": rf["unit"], "peak": rf["peak"],
                         "kernel_frac": rf["frac"], "step_frac": rf["step"]["frac"],
                         "traffic": rf["traffic"], "kernel_ms": rf["kernel_ms"]},
            "roofline_hbm": {"unit": rh["unit"], "peak": rh["peak"], "kernel_frac": rh["frac"],
                             "step_frac": rh["step"]["frac"],
                             "step_achieved": rh["step"]["achieved"]},
            "launch_ms": ln["launch_ms"],
            "plan": ln["plan"],
            "gpu_launches": ln["gpu_launches"],
            "clocks": r.get("clocks"),
        }
        if not args.no_cpu_baseline:
            import oracle
            threads = oracle.max_threads()
            cfg = workload_config(name)
            v, desc, _ = cpu_baseline_parallel(cfg, args.per_config_cpu_seconds, threads)
            summary["cpu_baseline"] = {"value": v, "unit": "updates/s", "cores": threads,
                                       "kind": "oracle", "sample": desc}
        out[name] = summary
    return out if rank == 0 else None


def run_front(args, rank, world, local_rank):
    """The fused front + scan (selective_scan_fwd_front) of the Vim-S block:
    one step = conv1d + SiLU + x_proj (tensor cores) + dt_proj of both
    directions, their scans and the sum, inputs resident in HBM, L2 flushed
    before every timed step.  Returns the JSON line (rank 0)."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from selective_scan_ss2d_b200 import binding
    from selective_scan_ss2d_b200 import workloads as wl

    cfg = wl.FRONT_CONFIGS[args.front_config]
    if args.dtype:
        cfg = cfg.with_(dtype=args.dtype)
    dev = torch.device(f"cuda:{local_rank}")
    torch.cuda.set_device(dev)
    binding.lib()
    inp = wl.make_front_inputs(cfg, seed=rank)
    tdt = {wl.F32: torch.float32, wl.BF16: torch.bfloat16, wl.F16: torch.float16}[cfg.dtype]
    x = (torch.from_numpy(inp.x.view(np.int16)).view(torch.bfloat16) if inp.x.dtype == np.uint16
         else torch.from_numpy(inp.x)).to(dev)
    assert x.dtype == tdt
    wts = {n: torch.from_numpy(getattr(inp, n)).to(dev) for n in wl.FrontInputs.WEIGHTS}
    y = torch.empty((cfg.B, cfg.D, cfg.L), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024) or 126 * 1024 * 1024
    flush = torch.empty(int(2 * l2) // 4, dtype=torch.float32, device=dev)
    args_f = [x] + [wts[n] for n in wl.FrontInputs.WEIGHTS]

    def step():
        binding.selective_scan_fwd_front(*args_f, y)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    gpu_id = str(getattr(props, "uuid", local_rank))
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) >= 32:
        gpu_id = "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.2)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push(f"front {cfg.name} timed steps")
    for i in range(args.steps):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev)
    value = whole_job_rate(cfg.updates, args.steps, world, total_ms)
    per = []
    for i in range(args.steps):
        flush.fill_(float(i))
        per.append(binding.selective_scan_fwd_front_timed(*args_f, y, stream=stream.cuda_stream))
    front_ms = statistics.mean(r[0] for r in per)
    scan_ms = statistics.mean(r[1] for r in per)
    merge_ms = statistics.mean(r[2] for r in per if r[2] >= 0) if cfg.K > 1 else None
    if rank != 0:
        return None
    peaks = measured_peaks()
    esz = 4 if cfg.dtype == wl.F32 else 2
    R = 1 + 2 * cfg.N
    # x_proj on the tensor cores: useful flops (M = steps, N = 1 + 2N, K = D)
    flops = 2.0 * cfg.B * cfg.K * cfg.L * cfg.D * R
    # the front kernel's algorithmic bytes: x read once per direction, u
    # written once (input dtype), dt_raw, B, C written once (float32), weights
    front_bytes = (cfg.K * cfg.B * cfg.L * cfg.D * esz + cfg.B * cfg.K * cfg.D * cfg.L * esz +
                   cfg.B * cfg.K * cfg.L * R * 4 + cfg.K * cfg.D * (4 + 1 + R + 1) * 4)
    # the whole call's algorithmic bytes: x read once, y written once, weights
    step_bytes = (cfg.B * cfg.L * cfg.D * esz + cfg.B * cfg.D * cfg.L * 4 +
                  cfg.K * cfg.D * (4 + 1 + R + 1 + cfg.N + 2) * 4)
    step_s = total_ms / args.steps / 1e3
    exps = cfg.updates + cfg.B * cfg.K * cfg.D * cfg.L
    mufu_peak = NUM_SMS * MUFU_EX2_PER_CLK_PER_SM * peaks["sm_max_mhz"] * 1e6 / 1e9
    tflops = flops / (front_ms / 1e3) / 1e12
    front_gbs = front_bytes / (front_ms / 1e3) / 1e9
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "updates/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded N(0,1) input branch and unit-scale weights)",
        "config": {"workload": cfg.name, "B": cfg.B, "L": cfg.L, "D": cfg.D, "N": cfg.N,
                   "K": cfg.K, "input_dtype": cfg.dtype, "entry": "selective_scan_fwd_front",
                   "l2": "flushed before every timed step (2x L2 write, outside events)",
                   "parallelism": f"replicas x{world}"},
        "roofline_front_tensor": {"bound": "tensor", "achieved": tflops,
                                  "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                  "frac": tflops / peaks["bf16_tflops"],
                                  "kernel": "front_conv_kernel (with the W_x conversion) + "
                                            "front_proj_kernel (x_proj on tcgen05, bf16 operands)",
                                  "kernel_ms": front_ms, "flops_per_launch": flops,
                                  "peak_source": peaks["bf16_source"]},
        "roofline_front_hbm": {"bound": "hbm", "achieved": front_gbs, "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": front_gbs / peaks["hbm_gbs"],
                               "bytes_per_launch": front_bytes, "kernel_ms": front_ms,
                               "peak_source": f"{peaks['source']} (hbm_gbs)"},
        "roofline": {"bound": "alu", "unit": "Gexp2/s", "peak": mufu_peak,
                     "achieved": exps / (scan_ms / 1e3) / 1e9,
                     "frac": exps / (scan_ms / 1e3) / 1e9 / mufu_peak,
                     "kernel": "lane_scan_kernel passes on the front's outputs",
                     "kernel_ms": scan_ms,
                     "step": {"achieved": exps / step_s / 1e9,
                              "frac": exps / step_s / 1e9 / mufu_peak}},
        "roofline_hbm": {"bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                         "step": {"achieved": step_bytes / step_s / 1e9,
                                  "frac": step_bytes / step_s / 1e9 / peaks["hbm_gbs"]},
                         "algorithmic_bytes_per_step": step_bytes},
        "launch_ms": {"front": front_ms, "scan_passes": scan_ms, "cross_merge": merge_ms},
        # two front kernels, then the front-mode scan's own launches (its
        # passes and the merge) under the lane kernel's plan
        "gpu_launches": args.steps * (2 + front_scan_launches(cfg)),
        "clocks": clocks,
    }
    return line


def front_scan_launches(cfg) -> int:
    """Kernel launches of the scan + merge half of one selective_scan_fwd_front
    call: the plan of the lane kernel's wave-chunked variant, which that call
    always uses."""
    from selective_scan_ss2d_b200 import binding
    names = [binding.ss2d_variant_name(i) for i in range(binding.ss2d_num_variants())]
    plan = binding.ss2d_plan(False, cfg.B, cfg.D, 1, cfg.L, cfg.N, cfg.K,
                             variant=names.index("lane2_wave"))
    return plan["launches"]


def run_backward(args, rank, world, local_rank):
    """The backward pass (ss2d_backward / selective_scan_bwd) of the workload:
    one step = the gradients of every input for one seeded cotangent, inputs
    resident in HBM, L2 flushed before every timed step.  Returns the JSON
    line (rank 0) with the exp-unit roofline of the whole call."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from selective_scan_ss2d_b200 import binding
    from selective_scan_ss2d_b200 import workloads as wl

    cfg = workload_config(args.config, args.dtype, args.n_states)
    dev = torch.device(f"cuda:{local_rank}")
    torch.cuda.set_device(dev)
    binding.lib()
    inp, t = build_arrays(cfg, seed=rank, device=dev)
    dy = torch.from_numpy(wl.make_cotangent(cfg, seed=rank)).to(dev)
    fn = binding.ss2d_backward if cfg.kind == "2d" else binding.selective_scan_bwd
    stream = torch.cuda.current_stream(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024) or 126 * 1024 * 1024
    flush = torch.empty(int(2 * l2) // 4, dtype=torch.float32, device=dev)

    label = f"ss2d backward {cfg.name}"

    def step():
        return fn(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"],
                  dy, stream=stream.cuda_stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    gpu_id = str(getattr(props, "uuid", local_rank))
    if gpu_id and not gpu_id.startswith("GPU-") and len(gpu_id) >= 32:
        gpu_id = "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.2)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push(f"{label} timed steps")   # marks the region for a trace
    for i in range(args.steps):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev)
    value = whole_job_rate(cfg.updates, args.steps, world, total_ms)
    if rank != 0:
        return None
    peaks = measured_peaks()
    step_s = total_ms / args.steps / 1e3
    mufu_peak = NUM_SMS * MUFU_EX2_PER_CLK_PER_SM * peaks["sm_max_mhz"] * 1e6 / 1e9
    bkdl = cfg.B * cfg.K * cfg.D * cfg.L
    exps = 2 * cfg.updates + 2 * bkdl            # recompute + reverse walk; softplus + sigmoid
    exps_done = (4 * cfg.updates + 4 * bkdl) if cfg.L > 16 else exps
    in_b = cfg.in_bytes_per_elem
    nbc = cfg.B * cfg.K * cfg.N * cfg.L
    grad_bytes = (cfg.B * cfg.D * cfg.L * (in_b + 4 + 4) + bkdl * (in_b + 4) + nbc * 2 * (in_b + 4))
    return {
        "metric": "SS2D backward: state updates/s (B·K·D·L·N) of the gradient pass",
        "value": value, "unit": "updates/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) inputs and cotangent)",
        "config": {"workload": cfg.name, "B": cfg.B, "D": cfg.D, "H": cfg.H, "W": cfg.W,
                   "L": cfg.L, "K": cfg.K, "N": cfg.N, "input_dtype": cfg.dtype,
                   "pass": "backward (all seven gradients)",
                   "l2": "flushed before every timed step (2x L2 write, outside events)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "alu", "achieved": exps / step_s / 1e9, "peak": mufu_peak,
                     "unit": "Gexp2/s", "frac": exps / step_s / 1e9 / mufu_peak,
                     "work": "2 exp2 per state update (recompute, reverse walk) + 2 per "
                             "(b,k,d,l) (softplus, sigmoid); this implementation issues "
                             f"{exps_done / exps:.2f}x that (the chunk-local pass)",
                     "peak_source": f"MUFU exp2 x {peaks['sm_max_mhz']:.0f} MHz ({peaks['source']})"},
        "roofline_hbm": {"bound": "hbm", "achieved": grad_bytes / step_s / 1e9,
                         "peak": peaks["hbm_gbs"],
                         "frac": grad_bytes / step_s / 1e9 / peaks["hbm_gbs"],
                         "unit": "GB/s", "bytes": "inputs and dy read once, gradients written once"},
        "clocks": clocks,
    }


def run_e2e(args, cfg_name, local_rank, world=1):
    """Same metric through the C ABI with host (pinned) buffers: every step
    copies the inputs in, computes, and copies y out, inside the call.  Every
    rank runs it; the slowest rank's time counts."""
    import torch
    from selective_scan_ss2d_b200 import binding
    from selective_scan_ss2d_b200 import workloads as wl
    cfg = workload_config(cfg_name, args.dtype, args.n_states)
    dev = torch.device(f"cuda:{local_rank}")
    inp, t = build_arrays(cfg, seed=0, device=None, pin=True)
    y = torch.empty(inp.x.shape, dtype=torch.float32).pin_memory()
    fn = binding.ss2d_forward if cfg.kind == "2d" else binding.selective_scan_fwd
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(1, min(args.warmup, 3))):
        fn(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"], y,
           stream=stream.cuda_stream, variant=args.variant)
    n = max(3, min(args.steps, 20))
    evs = []
    torch.cuda.nvtx.range_push(f"ss2d forward end to end {cfg.name}")
    for _ in range(n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn(t["x"], t["delta"], t["A_log"], t["Bs"], t["Cs"], t["Dskip"], t["delta_bias"], y,
           stream=stream.cuda_stream, variant=args.variant)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    total = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), dev)
    h2d = sum(getattr(inp, nm).nbytes for nm in wl.Inputs.STREAMED + wl.Inputs.PARAMS)
    d2h = y.numel() * 4
    return {"value": whole_job_rate(cfg.updates, n, world, total), "unit": "updates/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": total / n,
            "steps": n}


def run_reference(args):
    """The float64 oracle on the host cores: each step is a bounded sample
    (whole channels of batch element 0) of the workload."""
    import oracle
    from selective_scan_ss2d_b200 import workloads as wl
    cfg = workload_config(args.config, args.dtype, args.n_states)
    threads = oracle.max_threads()
    # size one step to ~ (budget / (steps + warmup)) seconds of host work
    budget_s = float(os.environ.get("SS2D_REFERENCE_BUDGET_S", "150"))
    per_step_s = max(0.5, min(10.0, budget_s / max(1, args.steps + args.warmup)))
    _, desc, _ = cpu_baseline_parallel(cfg, per_step_s, threads)
    nb = int(desc.split("batch elements 0..")[1].split(",")[0]) + 1
    nd = int(desc.split("channels 0..")[1].split(" ")[0]) + 1
    inp = wl.make_inputs(cfg, seed=0)
    sub = slice_sample(inp, nb, nd)
    ff = sub.as_f64()
    fn = oracle.ss2d_forward if cfg.kind == "2d" else oracle.selective_scan_fwd

    def step():
        fn(ff["x"], ff["delta"], ff["A_log"], ff["Bs"], ff["Cs"], ff["Dskip"], ff["delta_bias"],
           K=cfg.K, threads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    upd = sub.cfg.updates
    value = upd * args.steps / dt
    sample = (f"per step: batch elements 0..{nb - 1}, channels 0..{nd - 1} of {cfg.D}, all "
              f"{cfg.K} directions over the full L={cfg.L} ({upd} updates)")
    return {
        "metric": METRIC, "value": value, "unit": "updates/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": cfg.name, "B": cfg.B, "D": cfg.D, "H": cfg.H, "W": cfg.W,
                   "K": cfg.K, "N": cfg.N, "input_dtype": cfg.dtype},
        "cpu_baseline": {"value": value, "unit": "updates/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "updates/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--variant", type=int, default=-1)
    ap.add_argument("--dtype", choices=["f32", "bf16", "f16"], default=None,
                    help="storage dtype of x, delta, Bs, Cs (default: the workload's own)")
    ap.add_argument("--n-states", type=int, default=None,
                    help="state count N, 1..64 (default: the workload's own, 16)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="host seconds for the oracle sample of cpu_baseline")
    ap.add_argument("--gate", action="store_true",
                    help="time the gated entry point (y * SiLU(z)); device buffers only, "
                         "so no e2e leg")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (gradients of every input) instead; "
                         "device buffers only, no e2e or CPU leg")
    ap.add_argument("--front", action="store_true",
                    help="time the fused front + scan (selective_scan_fwd_front) instead")
    ap.add_argument("--front-config", default="vim_s_front")
    ap.add_argument("--no-per-config", action="store_true",
                    help="leave out the per_config summaries of the other workloads")
    ap.add_argument("--per-config-steps", type=int, default=10,
                    help="timed steps of each per_config workload")
    ap.add_argument("--per-config-cpu-seconds", type=float, default=3.0,
                    help="host seconds for each per_config oracle sample")
    ap.add_argument("--report", action="store_true",
                    help="one JSON line per workload (device-resident only)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.n_states is not None and not 1 <= args.n_states <= 64:
        ap.error("--n-states must be in 1..64")
    if args.n_states and args.n_states > 16 and not args.backward and args.impl == "ours":
        # the per-launch timing of the forward line covers one group of 16 states
        ap.error("the forward bench takes --n-states up to 16 (--backward takes up to 64)")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    init_distributed(world, local_rank)

    if args.front:
        line = run_front(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return 0

    if args.backward:
        line = run_backward(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return 0

    if args.report:
        from selective_scan_ss2d_b200 import workloads as wl
        for name in wl.CONFIG_ORDER:
            a = argparse.Namespace(**vars(args))
            a.config = name
            r = run_ours(a, rank, world, local_rank)
            if rank == 0:
                line = r["line"]
                line["clocks"] = r.get("clocks")
                print(json.dumps(line), flush=True)
        return 0

    r = run_ours(args, rank, world, local_rank)
    e2e = None if (args.no_e2e or args.gate) else run_e2e(args, args.config, local_rank, world)
    per_config = None
    if world == 1 and not args.no_per_config:
        per_config = run_per_config(args, rank, world, local_rank)
    if rank == 0:
        line = r["line"]
        line["clocks"] = r.get("clocks")
        if e2e is not None:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            from selective_scan_ss2d_b200 import workloads as wl
            cfg = workload_config(args.config, args.dtype, args.n_states)
            threads = oracle.max_threads()
            v, desc, _ = cpu_baseline_parallel(cfg, args.cpu_seconds, threads)
            line["cpu_baseline"] = {"value": v, "unit": "updates/s", "cores": threads,
                                    "kind": "oracle", "sample": desc}
        if per_config is not None:
            line["per_config"] = per_config
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

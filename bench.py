"""Benchmark of the routed-expert MoE layer on 4-bit block-scaled weights (B200).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config all|NAME]

Default (--config all): every workload on each GPU, reported as ONE JSON line. The
top-level keys are the headline workload, the largest single-GPU configuration: the
MXFP4 MoE prefill layer (8192 bf16 tokens, 256 experts, hidden 6144, expert
intermediate 2048, top-8). "workloads" holds the same record for the other seven:
the dense MXFP4 W4A16 linear layer (16 x 2048 x 2048), the MXFP4 decode layer (64
experts, hidden 2048, intermediate 768, top-8, 16 tokens), the NVFP4 decode layer
(256 experts, hidden 6144, intermediate 2048, 64 tokens, Zipf-skewed router), the CB4
codebook-plus-outlier decode layer (the MXFP4 decode layer's dimensions), the NVFP4
prefill layer (the MXFP4 prefill layer's dimensions), the V2a shared-library decode layer
and a mixed buffer of MXFP4 and bf16 experts (both at the MXFP4 decode layer's
dimensions).  Each record carries its roofline (dominant kernel's device time per launch,
algorithmic bytes or flops, DRAM traffic from the committed ncu summary of the same
kernel sources), e2e, clocks, launch count and CPU-oracle baseline.

One step = one full layer call (router, gate_up + fused SwiGLU-with-clamp, down,
weighted combine; for the linear layer one y = x W^T) on device-resident inputs,
replayed from CUDA graphs. Metric: decode = HBM GB/s of algorithmic bytes (codes +
scales of every expert the step routes to, once, + router weights + x + y); prefill =
TFLOP/s of 6 T k H I dense-equivalent flops (and tokens/s).

Multi-GPU (torchrun): every rank runs an independent replica of each workload
("replicas only": nothing is sharded), each timed region is bracketed by a barrier and
a device synchronisation on both sides, and the slowest rank's time is reported:
value = all ranks' work / that time.

--impl reference times the CPU oracle (float64 numpy) on a bounded sample of the
headline workload: each step runs one routed (token, expert) pair of the first token.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import functools
import glob
import hashlib
import json
import multiprocessing as mp
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import configs as C, draws as D  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "FP4 MoE layer: decode HBM GB/s (% of peak); prefill TFLOP/s; tokens/s"
HEADLINE = C.MOE_C4.name
ORDER = [C.MOE_C4.name, C.LINEAR_C1.name, C.MOE_C2.name, C.MOE_C3.name, C.MOE_C5.name, C.MOE_C4_NV.name,
         C.MOE_C5_V2A.name, C.MOE_C2_MIXED.name]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="all", choices=["all"] + sorted(C.FULL) + sorted(C.PROFILE))
    ap.add_argument("--variant", type=int, default=0, choices=[0, 1, 2],
                    help="expert kernels: 0 chosen by the library, 1 CUDA-core GEMV, 2 tensor cores")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed CPU oracle samples")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle time per CPU baseline")
    return ap.parse_args(argv)


# ------------------------------------------------------------------------------------
# work accounting (closed forms; pinned by tests/test_bench_metrics.py)
# ------------------------------------------------------------------------------------
def per_expert_bytes(cfg):
    """Dense bytes of one expert (all matrices, gate_up only): codes + scales; CB4 counts
    indices + fp16 codebooks here and its CSR per expert separately (cb4_extra_bytes)."""
    gu = 2 * cfg.I * cfg.H
    dn = cfg.H * cfg.I
    if cfg.fmt == "cb4":
        return (gu + dn) // 2 + (gu + dn) // 4, gu // 2 + gu // 4
    if cfg.fmt == "v2a":       # 4-bit codes + an 8-byte record per 128 weights + a 1 KB library per matrix
        return (gu + dn) // 2 + (gu + dn) // 16 + 2 * 1024, gu // 2 + gu // 16 + 1024
    B = 32 if cfg.fmt in ("mxfp4", "mixed") else 16       # mixed: the MXFP4 experts (bf16 ones via extra)
    b = (gu + dn) // 2 + (gu + dn) // B
    if cfg.fmt == "nvfp4":
        b += 8
    return b, gu // 2 + gu // B + (4 if cfg.fmt == "nvfp4" else 0)


def is_prefill(cfg):
    return "prefill" in cfg.name


def layer_flops(cfg, tokens=None):
    """Dense-equivalent flops of the routed experts: 2 T k (2I H + H I) = 6 T k H I."""
    T = cfg.T if tokens is None else tokens
    return 6 * T * cfg.k * cfg.H * cfg.I


def work_per_step(cfg, counts, tokens=None, extra=None):
    """Amount of the metric's work in one step and its rate unit: prefill counts
    TFLOP, decode counts GB of algorithmic bytes."""
    if is_prefill(cfg):
        return layer_flops(cfg, tokens) / 1e12, "TFLOP/s"
    return algorithmic_bytes(cfg, counts, tokens, extra) / 1e9, "GB/s"


def linear_bytes(cfg):
    """Dense linear layer: codes + scales (+ tensor scale) + x + y."""
    B = 32 if cfg.fmt == "mxfp4" else 16
    return cfg.N * cfg.K // 2 + cfg.N * cfg.K // B + (4 if cfg.fmt == "nvfp4" else 0) + 2 * cfg.T * (cfg.K + cfg.N)


def cb4_extra_bytes(w):
    """CB4 sparse term per expert: (gate_up, all) bytes of CSR values, columns and row
    pointers, from the packed weights."""
    out = []
    for rp, rows in ((w.gu_rowptr, 2 * w.I), (w.dn_rowptr, w.H)):
        r = rp.cpu().numpy().astype(np.int64)
        nnz = r[rows::rows] - r[:-1:rows][:w.E]
        out.append(nnz * 6 + 4 * rows)
    return out[0], out[0] + out[1]


def algorithmic_bytes(cfg, counts, tokens=None, extra=None):
    """Active-bytes rule: every routed expert's weight bytes once + router + x + y
    (extra: per-expert bytes beyond the dense part, counted for routed experts)."""
    per, _ = per_expert_bytes(cfg)
    d = int(np.count_nonzero(counts))
    T = cfg.T if tokens is None else tokens
    router = cfg.E * cfg.H * 4 + (cfg.E * 4 if cfg.zipf_bias else 0)
    more = 0 if extra is None else int(np.sum(np.asarray(extra)[np.asarray(counts) > 0]))
    return d * per + more + router + 2 * T * cfg.H * 2


def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank timings over all ranks (the slowest replica sets
    the job's time); identity on one rank."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_rate(work_per_rank, world, ms):
    """Whole-job rate: the work of every replica over the slowest replica's time."""
    return work_per_rank * world / (ms * 1e-3)


# ------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, enabled=True):
        self.index = index
        self.enabled = enabled
        self.proc = None
        self.lines = []

    def start(self):
        if not self.enabled:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.enabled:
            return None
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------
# peaks and ncu traffic
# ------------------------------------------------------------------------------------
def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def measure_block_scaled_peaks(device):
    """Dense block-scaled GEMM throughput of the vendor library on this GPU (torch's
    scaled_mm over cuBLASLt), M = N = K = 8192, 20 timed calls after 3: FP4 E2M1 with
    UE8M0 scales per 32 (MXFP4), with E4M3 scales per 16 (NVFP4), and E4M3 with UE8M0
    per 32 (MXFP8).  TFLOP/s; a format the library refuses is reported as null."""
    import torch
    import torch.nn.functional as F
    try:
        from torch.nn.functional import ScalingType, SwizzleType
    except ImportError:
        return {"mxfp4": None, "nvfp4": None, "mxfp8": None, "note": "torch has no scaled_mm recipes"}
    n = 8192
    ru = lambda a, b: (a + b - 1) // b * b
    out = {}
    specs = {"mxfp4": (torch.float4_e2m1fn_x2, 2, 32, torch.float8_e8m0fnu, 127, ScalingType.BlockWise1x32),
             "nvfp4": (torch.float4_e2m1fn_x2, 2, 16, torch.float8_e4m3fn, 0x38, ScalingType.BlockWise1x16),
             "mxfp8": (torch.float8_e4m3fn, 1, 32, torch.float8_e8m0fnu, 127, ScalingType.BlockWise1x32)}
    for name, (dt, per_byte, blk, sdt, sval, rec) in specs.items():
        try:
            hi = 256 if per_byte == 2 else 120            # E4M3 bytes below 0x78: finite, |v| <= 240
            a = torch.randint(0, hi, (n, n // per_byte), device=device, dtype=torch.uint8).view(dt)
            b = torch.randint(0, hi, (n, n // per_byte), device=device, dtype=torch.uint8).view(dt)
            sa = torch.full((ru(n, 128) * ru(n // blk, 4),), sval, device=device, dtype=torch.uint8).view(sdt)
            sb = torch.full((ru(n, 128) * ru(n // blk, 4),), sval, device=device, dtype=torch.uint8).view(sdt)
            fn = lambda: F.scaled_mm(a, b.t(), sa, rec, sb, rec, SwizzleType.SWIZZLE_32_4_4,
                                     SwizzleType.SWIZZLE_32_4_4, output_dtype=torch.bfloat16)
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(20):
                fn()
            e1.record()
            torch.cuda.synchronize()
            out[name] = 2.0 * n ** 3 / (e0.elapsed_time(e1) / 20 * 1e-3) / 1e12
            del a, b, sa, sb
        except Exception as ex:                       # library refuses the format on this build
            out[name] = None
            out[name + "_error"] = repr(ex)[:160]
    torch.cuda.empty_cache()
    out["how"] = "torch scaled_mm (cuBLASLt), 8192^3, burst of 20 calls"
    return out


KERNEL_SOURCES = {
    "bs_moe_kernel": ["bs_moe.cu", "tcgen05.cuh", "common.cuh", "kernels.cuh"],
    "nv_moe_kernel": ["nv_moe.cu", "tcgen05.cuh", "common.cuh", "kernels.cuh"],
    "decode_kernel": ["decode.cu", "common.cuh", "kernels.cuh", "routing.cuh"],
}


def kernel_source_hash(kernel):
    base = kernel.split("<")[0]
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(base, []):
        with open(os.path.join(ROOT, "fp4_block_scaled_moe_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def profile_traffic(workload, kernel):
    """DRAM bytes (read + write) per launch of ``kernel`` on ``workload`` from a committed
    ncu summary under profiles/ (a line "bench-traffic: workload=... kernel=...
    bytes_per_launch=... sources=<hash>"); None when there is none or when the kernel's
    sources have changed since that capture (hash mismatch)."""
    want = kernel_source_hash(kernel)
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(path, encoding="utf-8") as f:
            for line in f:
                m = re.search(r"bench-traffic:\s*workload=(\S+)\s+kernel=(\S+)\s+bytes_per_launch=(\d+)\s+"
                              r"sources=([0-9a-f]+)", line)
                if m and m.group(1) == workload and m.group(2) == kernel and m.group(4) == want:
                    return int(m.group(3)), os.path.relpath(path, ROOT)
    return None, None


# ------------------------------------------------------------------------------------
# timing helpers
# ------------------------------------------------------------------------------------
def timed_replays(graphs, steps, stream, world, clk):
    """CUDA-event time (ms) of ``steps`` graph replays (cycling ``graphs``), bracketed by a
    barrier and a device synchronisation on both sides."""
    import torch
    import torch.distributed as dist
    clk.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        with torch.cuda.stream(stream):
            graphs[i % len(graphs)].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clk.stop()
    return e0.elapsed_time(e1), clocks


def capture(fn, stream):
    """One CUDA graph of fn() (called once untimed first); returns (graph, library launches)."""
    import torch
    from fp4_block_scaled_moe_b200 import api
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()
        torch.cuda.synchronize()
        n0 = api.fp4_launch_count()
        with torch.cuda.graph(g, stream=stream):
            fn()
        n = api.fp4_launch_count() - n0
    return g, n


# ------------------------------------------------------------------------------------
# MoE layers
# ------------------------------------------------------------------------------------
def clone_weights(w0, copies):
    import dataclasses
    import torch
    out = [w0]
    for _ in range(copies - 1):
        out.append(dataclasses.replace(w0, **{f.name: getattr(w0, f.name).clone() for f in dataclasses.fields(w0)
                                              if isinstance(getattr(w0, f.name), torch.Tensor)}))
    return out


def run_moe(args, cfg, device, world, peaks):
    import torch
    from fp4_block_scaled_moe_b200 import api, prepare_mma_scales
    from fp4_block_scaled_moe_b200.workloads import device_weights
    per, _ = per_expert_bytes(cfg)
    bank_bytes = per * cfg.E
    copies = max(2, int(np.ceil(2 * L2_BYTES / bank_bytes)) + 1) if bank_bytes < 4 * L2_BYTES else 1
    w0 = device_weights(cfg, device=device)
    w0.kernel_variant = args.variant
    if cfg.fmt in ("mxfp4", "nvfp4") and args.variant != 1:
        prepare_mma_scales(w0)            # one-time weight preparation, outside the timed region
    elif cfg.fmt == "mixed" and args.variant != 0:
        w0.kernel_variant = args.variant
    weights = clone_weights(w0, copies)
    structs = [w.c_struct() for w in weights]
    T, k = cfg.T, cfg.k
    kernels = api.moe_fp4_expert_kernels(w0, T, k)
    x_bits = D.activations_bf16(cfg.seed, T, cfg.H)
    wr = torch.from_numpy(D.router_weights(cfg.seed, cfg.E, cfg.H)).to(device)
    bias = torch.from_numpy(D.zipf_bias(cfg.seed, cfg.E)).to(device) if cfg.zipf_bias else None
    x = torch.from_numpy(x_bits.view(np.int16)).to(device).view(torch.bfloat16)
    ws = api.alloc_workspace(api.moe_fp4_workspace_size(w0, T, k), device)
    y = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=device)
    route = {"counts": torch.empty(cfg.E, dtype=torch.int32, device=device)}
    stream = torch.cuda.Stream(device)

    def step(i, r=None):
        api.moe_fp4_forward(weights[i % copies], x, wr, bias, k, workspace=ws, y=y, _struct=structs[i % copies],
                            route_out=r)

    with torch.cuda.stream(stream):
        step(0, route)
    torch.cuda.synchronize()
    counts = route["counts"].cpu().numpy()
    extra_gu = extra_all = None
    if cfg.fmt in ("cb4", "v2a"):
        extra_gu, extra_all = cb4_extra_bytes(w0)
    if cfg.fmt == "mixed":           # bf16 experts move 2 bytes per weight instead of the MXFP4 bytes
        gu_d = 2 * (2 * cfg.I * cfg.H) - per_expert_bytes(cfg)[1]
        all_d = 2 * (3 * cfg.I * cfg.H) - per_expert_bytes(cfg)[0]
        extra_gu = np.array([gu_d if e in cfg.bf16_experts else 0 for e in range(cfg.E)], dtype=np.int64)
        extra_all = np.array([all_d if e in cfg.bf16_experts else 0 for e in range(cfg.E)], dtype=np.int64)
    work_step, unit = work_per_step(cfg, counts, extra=extra_all)
    graphs, launches = [], 0
    for c in range(copies):
        g, launches = capture(functools.partial(step, c), stream)
        graphs.append(g)
    for i in range(args.warmup):
        with torch.cuda.stream(stream):
            graphs[i % copies].replay()
    torch.cuda.synchronize()
    api.fp4_workspace_kernel_stats(ws, reset=True)
    clk = ClockSampler(device.index or 0, not args.no_clocks)
    ms_total, clocks = timed_replays(graphs, args.steps, stream, world, clk)
    kern = api.fp4_workspace_kernel_stats(ws)
    status = api.fp4_workspace_status(ws)
    del graphs

    # end to end through the public API: pinned x -> device, layer, y -> pinned host each step
    x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((T, cfg.H), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)

    def e2e_step(i):
        with torch.cuda.stream(stream):
            x_dev.copy_(x_host, non_blocking=True)
            api.moe_fp4_forward(weights[i % copies], x_dev, wr, bias, k, workspace=ws, y=y,
                                _struct=structs[i % copies])
            y_host.copy_(y, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a0.elapsed_time(a1)
    gu_ms = kern["gate_up_ns"] / max(kern["gate_up_launches"], 1) / 1e6
    dn_ms = kern["down_ns"] / max(kern["down_launches"], 1) / 1e6
    ms_total, e2e_ms, gu_ms, dn_ms = max_over_ranks([ms_total, e2e_ms, gu_ms, dn_ms], world, device)
    ms_step = ms_total / args.steps
    value = job_rate(work_step, world, ms_step)
    tensor = kernels == 2
    hbm = peaks.get("hbm_gbs", 6650.0)
    conf = {"workload": cfg.name, "tokens": T, "experts": cfg.E, "hidden": cfg.H, "inter": cfg.I, "top_k": k,
            "format": cfg.fmt, "parallelism": f"replicas{world}",
            "l2": (f"weights rotate over {copies} copies ({copies * bank_bytes / 1e6:.0f} MB) > L2" if copies > 1
                   else f"weights {bank_bytes / 1e6:.0f} MB > L2, one copy"),
            "distinct_experts": int(np.count_nonzero(counts)), "max_tokens_per_expert": int(counts.max()),
            "expert_kernels": "tensor-core block-scaled" if tensor else "CUDA-core grouped GEMV",
            "bytes_per_step": int(algorithmic_bytes(cfg, counts, extra=extra_all))}
    if is_prefill(cfg):
        conf["tokens_per_s"] = T * world / (ms_step * 1e-3)
        conf["pct_of_bf16_measured_peak"] = 100 * value / world / peaks.get("bf16_tflops", 1590.0)
    else:
        conf["pct_of_hbm_peak"] = 100 * value / world / hbm
        conf["pct_of_hbm_spec_8000"] = 100 * value / world / 8000.0
    kern_ms = {"gate_up": gu_ms, "down": dn_ms}
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype_label(cfg, tensor),
        "data": "synthetic", "config": conf,
        "e2e": {"value": job_rate(work_step, world, e2e_ms / args.steps), "unit": unit,
                "h2d_bytes_per_step": T * cfg.H * 2, "d2h_bytes_per_step": T * cfg.H * 2},
        "gpu_launches": launches * args.steps,
        "roofline": moe_roofline(cfg, counts, extra_gu, kern_ms, tensor, peaks),
        "clocks": clocks, "device_status": status,
    }
    del weights, ws
    torch.cuda.empty_cache()
    return line


def dtype_label(cfg, tensor):
    """Operand types of the expert MMAs the library ran -> accumulator type."""
    if cfg.fmt == "cb4":
        return "f16(codebook)xf16->f32"
    if cfg.fmt == "v2a":
        return "f16(shared-library codebook)xf16->f32"
    if cfg.fmt == "mixed":
        return "f16xe2m1->f32 and bf16xf16->f32 (fp32 FMA)"
    if tensor and cfg.fmt == "mxfp4":
        return "e4m3x2xe2m1->f32"
    return "f16xf16(e2m1*e4m3)->f32" if cfg.fmt == "nvfp4" else "f16xe2m1->f32"


def moe_roofline(cfg, counts, extra_gu, kern_ms, tensor, peaks):
    """Dominant kernel: gate_up with the fused SwiGLU, timed per launch on the device
    (globaltimer, accumulated in the workspace over the timed replays).
    Prefill: algorithmic flops per launch 4 T k H I against the measured bf16 peak (MXFP4:
    the two-term E4M3 x E2M1 MMAs run at the FP8 rate over twice the columns, so the bf16
    rate is their ceiling for these flops; NVFP4: f16 MMAs, the bf16 rate itself), also
    given against the measured FP4 / MXFP8 peaks.
    Decode: algorithmic bytes per launch = codes + scales of the gate_up rows of every
    routed expert + x read + h written."""
    ms = kern_ms["gate_up"]
    kname = ("nv_moe_kernel<gate_up+swiglu>" if cfg.fmt == "nvfp4" else "bs_moe_kernel<gate_up+swiglu>") if tensor \
        else "decode_kernel<gate_up+swiglu>"
    traffic, tsrc = profile_traffic(cfg.name, kname)
    base = {"kernel": kname, "ms_per_launch": ms, "down_ms_per_launch": kern_ms["down"], "traffic": traffic,
            "traffic_source": tsrc or "no ncu capture of the current kernel sources",
            "timer": "device globaltimer per launch, accumulated in the workspace over the timed steps"}
    if is_prefill(cfg):
        flops = 4 * cfg.T * cfg.k * cfg.H * cfg.I
        ach = flops / (ms * 1e-3) / 1e12 if ms > 0 else None
        peak = peaks.get("bf16_tflops", 1590.0)
        bs = peaks.get("_block_scaled", {})
        base.update({"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                     "frac": (ach / peak) if ach else None,
                     "peak_source": ("MEASURED_PEAKS.json bf16_tflops, burst (of measured)" if "bf16_tflops" in peaks
                                     else "fallback 1590 TFLOP/s bf16 (of fallback)"),
                     "frac_of_sustained": (ach / peaks["bf16_tflops_sustained"])
                     if ach and "bf16_tflops_sustained" in peaks else None,
                     "frac_of_fp4_measured": (ach / bs[cfg.fmt]) if ach and bs.get(cfg.fmt) else None,
                     "frac_of_mxfp8_measured": (ach / bs["mxfp8"]) if ach and bs.get("mxfp8") else None,
                     "frac_of_fp4_nominal_9000": (ach / 9000.0) if ach else None,
                     "flops_per_launch": int(flops)})
        return base
    _, gu_per_expert = per_expert_bytes(cfg)
    d = int(np.count_nonzero(counts))
    P = cfg.T * cfg.k
    if cfg.fmt == "mixed":
        # the GEMV reads the routed MXFP4 experts only (the bf16 ones run in dense16_kernel)
        d -= sum(1 for e in cfg.bf16_experts if counts[e] > 0)
        extra_gu = None
    alg = d * gu_per_expert + cfg.T * cfg.H * 2 + P * cfg.I * 2
    if extra_gu is not None:
        alg += int(np.sum(extra_gu[counts > 0]))
    ach = alg / (ms * 1e-3) / 1e9 if ms > 0 else None
    hbm = peaks.get("hbm_gbs", 6650.0)
    base.update({"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": (ach / hbm) if ach else None,
                 "peak_source": "MEASURED_PEAKS.json hbm_gbs (of measured)" if "hbm_gbs" in peaks
                 else "fallback 6650 GB/s (of fallback)", "bytes_per_launch": int(alg)})
    return base


# ------------------------------------------------------------------------------------
# the dense linear layer
# ------------------------------------------------------------------------------------
def run_linear(args, cfg, device, world, peaks):
    import torch
    from fp4_block_scaled_moe_b200 import api, fp4_pack
    w = torch.from_numpy(D.expert_weights(cfg.seed, C.TID_LINEAR, (cfg.N, cfg.K), sigma=cfg.sigma)).to(device)
    c0, s0, t0 = fp4_pack(w, cfg.fmt)
    del w
    wbytes = c0.numel() + s0.numel()
    copies = int(np.ceil(2 * L2_BYTES / wbytes)) + 1
    codes = c0.unsqueeze(0).repeat(copies, 1, 1).contiguous()
    scales = s0.unsqueeze(0).repeat(copies, 1, 1).contiguous()
    x_bits = D.activations_bf16(cfg.seed, cfg.T, cfg.K)
    x = torch.from_numpy(x_bits.view(np.int16)).to(device).view(torch.bfloat16)
    y = torch.empty((cfg.T, cfg.N), dtype=torch.bfloat16, device=device)
    ws = api.alloc_workspace(api.L.load().fp4_linear_workspace_size(cfg.T, cfg.K), device)
    stream = torch.cuda.Stream(device)
    # one graph replays one call per weight copy: a replay is `copies` steps over > 2 x L2 of weights
    per_graph = copies

    def calls():
        for i in range(per_graph):
            api.fp4_linear(x, codes[i], scales[i], t0, cfg.fmt, workspace=ws, y=y)

    g, launches = capture(calls, stream)
    for _ in range(max(1, args.warmup)):
        with torch.cuda.stream(stream):
            g.replay()
    torch.cuda.synchronize()
    api.fp4_workspace_kernel_stats(ws, reset=True)
    replays = max(1, int(np.ceil(args.steps / per_graph)))
    steps = replays * per_graph
    clk = ClockSampler(device.index or 0, not args.no_clocks)
    ms_total, clocks = timed_replays([g] * replays, replays, stream, world, clk)
    kern = api.fp4_workspace_kernel_stats(ws)
    status = api.fp4_workspace_status(ws)
    del g
    x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((cfg.T, cfg.N), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)

    def e2e_step(i):
        with torch.cuda.stream(stream):
            x_dev.copy_(x_host, non_blocking=True)
            api.fp4_linear(x_dev, codes[i % copies], scales[i % copies], t0, cfg.fmt, workspace=ws, y=y)
            y_host.copy_(y, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a0.elapsed_time(a1)
    k_ms = kern["gate_up_ns"] / max(kern["gate_up_launches"], 1) / 1e6
    ms_total, e2e_ms, k_ms = max_over_ranks([ms_total, e2e_ms, k_ms], world, device)
    b = linear_bytes(cfg)
    ms_step = ms_total / steps
    value = job_rate(b / 1e9, world, ms_step)
    hbm = peaks.get("hbm_gbs", 6650.0)
    kbytes = b                           # the kernel reads codes, scales and x (as f16) and writes y
    ach = kbytes / (k_ms * 1e-3) / 1e9 if k_ms > 0 else None
    traffic, tsrc = profile_traffic(cfg.name, "decode_kernel<linear>")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16xe2m1->f32", "data": "synthetic",
        "config": {"workload": cfg.name, "tokens": cfg.T, "n": cfg.N, "k": cfg.K, "format": cfg.fmt,
                   "parallelism": f"replicas{world}",
                   "l2": f"one graph of {per_graph} calls over {copies} weight copies ({copies * wbytes / 1e6:.0f} MB) > 2 x L2",
                   "bytes_per_step": b, "pct_of_hbm_peak": 100 * value / world / hbm},
        "e2e": {"value": job_rate(b / 1e9, world, e2e_ms / args.steps), "unit": "GB/s",
                "h2d_bytes_per_step": cfg.T * cfg.K * 2, "d2h_bytes_per_step": cfg.T * cfg.N * 2},
        "gpu_launches": launches * replays,
        "roofline": {"kernel": "decode_kernel<linear>", "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                     "frac": (ach / hbm) if ach else None,
                     "peak_source": "MEASURED_PEAKS.json hbm_gbs (of measured)" if "hbm_gbs" in peaks
                     else "fallback 6650 GB/s (of fallback)",
                     "bytes_per_launch": kbytes, "ms_per_launch": k_ms, "traffic": traffic,
                     "traffic_source": tsrc or "no ncu capture of the current kernel sources",
                     "timer": "device globaltimer per launch, accumulated in the workspace over the timed steps"},
        "clocks": clocks, "device_status": status,
    }
    del codes, scales, ws
    torch.cuda.empty_cache()
    return line


# ------------------------------------------------------------------------------------
# the CPU oracle: reference arm and cpu_baseline (bounded samples)
# ------------------------------------------------------------------------------------
def _limit_threads():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _quantise_expert(cfg, which, e):
    """Worker: the oracle's quantised form of one expert matrix (untimed preparation)."""
    from oracle import moe as M
    bank = M.LazyExpertBank(cfg.fmt, cfg.E, cfg.H, cfg.I, draw=functools.partial(C.expert_rows, cfg),
                            cb4_threshold=cfg.cb4_threshold_sigma * cfg.sigma, v2a_bits=cfg.v2a_bits,
                            bf16_experts=cfg.bf16_experts)
    return bank.packed(which, e)


def oracle_pairs(cfg):
    """The oracle's expert bank prepared for the first token's k routed experts (the
    quantisation, untimed, in a spawn process pool) and a function running the oracle on
    the j-th (token 0, expert) pair: router logits and top-k of token 0, then that
    expert's gate_up, SwiGLU-with-clamp and down.  Returns (run(j), work(j))."""
    from oracle import moe as M, routing as R
    x0 = D.bf16_bits_to_f32(D.activations_bf16(cfg.seed, cfg.T, cfg.H))[:1]
    wr = D.router_weights(cfg.seed, cfg.E, cfg.H)
    bias = D.zipf_bias(cfg.seed, cfg.E) if cfg.zipf_bias else None
    ids = R.topk(R.router_logits(x0, wr, bias), cfg.k)[0]
    bank = M.LazyExpertBank(cfg.fmt, cfg.E, cfg.H, cfg.I, draw=functools.partial(C.expert_rows, cfg),
                            cb4_threshold=cfg.cb4_threshold_sigma * cfg.sigma, v2a_bits=cfg.v2a_bits,
                            bf16_experts=cfg.bf16_experts)
    jobs = [(which, int(e)) for e in ids for which in ("gu", "dn")]
    with cf.ProcessPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1)),
                                mp_context=mp.get_context("spawn"), initializer=_limit_threads) as pool:
        for (which, e), packed in zip(jobs, pool.map(_quantise_expert, *zip(*[(cfg, w, e) for w, e in jobs]))):
            bank.preload(which, e, packed)
    per, _ = per_expert_bytes(cfg)
    csr = {}
    if cfg.fmt in ("cb4", "v2a"):
        for e in ids:
            csr[int(e)] = sum(6 * int(bank.packed(w, int(e))["row_ptr"][-1]) + 4 * r
                              for w, r in (("gu", 2 * cfg.I), ("dn", cfg.H)))

    def run(j):
        lg = R.router_logits(x0, wr, bias)
        R.topk(lg, cfg.k)
        M.expert_outputs(bank, int(ids[j % cfg.k]), x0, cfg.swiglu_limit)

    def work(j):
        if is_prefill(cfg):
            return 6 * cfg.H * cfg.I / 1e12
        return (per + csr.get(int(ids[j % cfg.k]), 0)) / 1e9

    return run, work


def linear_oracle(cfg):
    from oracle import formats as F, moe as M
    w = D.expert_weights(cfg.seed, C.TID_LINEAR, (cfg.N, cfg.K), sigma=cfg.sigma)
    packed = F.mxfp4_quantize(w) if cfg.fmt == "mxfp4" else F.nvfp4_quantize(w)
    x = D.bf16_bits_to_f32(D.activations_bf16(cfg.seed, cfg.T, cfg.K))

    def run(j):
        deq = F.mxfp4_dequantize(*packed) if cfg.fmt == "mxfp4" else F.nvfp4_dequantize(*packed)
        M.linear(x, deq)

    return run, lambda j: linear_bytes(cfg) / 1e9


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def sample_desc(cfg):
    if cfg.kind == "linear":
        return f"the whole {cfg.T}x{cfg.N}x{cfg.K} layer (dequantise + matmul)"
    return f"one (token, expert) pair per step: token 0's {cfg.k} routed experts in turn, of {cfg.T} tokens"


def cpu_baseline(cfg, budget_s):
    """The float64 oracle as it stands, timed on this host's cores on a bounded sample
    of the workload (about budget_s seconds), in the metric's unit."""
    run, work = linear_oracle(cfg) if cfg.kind == "linear" else oracle_pairs(cfg)
    run(0)                                             # warm (BLAS threads, page-in)
    done, reps, t0 = 0.0, 0, time.perf_counter()
    while True:
        run(reps)
        done += work(reps)
        reps += 1
        dt = time.perf_counter() - t0
        if dt > budget_s or reps >= 200:
            break
    unit = "GB/s" if cfg.kind == "linear" else work_per_step(cfg, np.ones(1))[1]
    return {"value": done / dt, "unit": unit, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{sample_desc(cfg)}; float64 numpy; {reps} steps in {dt:.1f} s"}


def run_reference(args, cfg, world):
    run, work = linear_oracle(cfg) if cfg.kind == "linear" else oracle_pairs(cfg)
    unit = "GB/s" if cfg.kind == "linear" else work_per_step(cfg, np.ones(1))[1]
    for j in range(args.warmup):
        run(j)
    done, t0 = 0.0, time.perf_counter()
    for j in range(args.steps):
        run(j)
        done += work(j)
    dt = time.perf_counter() - t0
    v = done / dt
    cb = {"value": v, "unit": unit, "cores": blas_threads(), "kind": "oracle",
          "sample": f"{sample_desc(cfg)}; float64 numpy"}
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "sample": sample_desc(cfg)}, "cpu_baseline": cb,
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------------------------
def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    names = ORDER if args.config == "all" else [args.config]
    allcfg = dict(C.FULL, **C.PROFILE)
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args, allcfg[names[0]], world)), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(device)
    peaks = measured_peaks()
    if any(is_prefill(allcfg[n]) for n in names):
        peaks["_block_scaled"] = measure_block_scaled_peaks(device)
    lines = {}
    for n in names:
        cfg = allcfg[n]
        lines[n] = (run_linear if cfg.kind == "linear" else run_moe)(args, cfg, device, world, peaks)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            lines[n]["cpu_baseline"] = cpu_baseline(cfg, args.cpu_budget)
    head = lines[names[0]]
    if "_block_scaled" in peaks:
        head["block_scaled_peaks_tflops"] = peaks["_block_scaled"]
    if len(names) > 1:
        head["workloads"] = {n: lines[n] for n in names[1:]}
    if rank == 0:
        print(json.dumps(head), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark of the routed-expert MoE layer on 4-bit block-scaled weights (B200).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

Default workload: the MXFP4 MoE decode layer (64 experts, hidden 2048, expert
intermediate 768, top-8 softmax router, 16 bf16 tokens). One step = one full
layer call (router, gate_up + fused SwiGLU-with-clamp, down, weighted combine)
on device-resident inputs. Metric: decode HBM GB/s = algorithmic bytes per step
(the active-bytes rule: codes + scales of every expert the step routes to,
router weights, x and y) / device time per step.

Multi-GPU (torchrun): every rank runs an independent replica of the layer
(expert weights are not sharded; "replicas only"), the K timed steps are
bracketed by a barrier and a device synchronisation on both sides, and the
slowest rank's time is reported: value = all ranks' bytes / that time.

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=C.MOE_C2.name, choices=sorted(C.FULL) + sorted(C.PROFILE))
    ap.add_argument("--variant", type=int, default=0, choices=[0, 1, 2],
                    help="expert kernels: 0 chosen by the library, 1 CUDA-core GEMV, 2 tensor cores (MXFP4)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed CPU oracle sample")
    return ap.parse_args()


def per_expert_bytes(cfg):
    """Dense bytes of one expert (all matrices, gate_up only): codes + scales; CB4 counts
    indices + fp16 codebooks here and its CSR per expert separately (cb4_extra_bytes)."""
    gu = 2 * cfg.I * cfg.H
    dn = cfg.H * cfg.I
    if cfg.fmt == "cb4":
        return (gu + dn) // 2 + (gu + dn) // 4, gu // 2 + gu // 4
    B = 32 if cfg.fmt == "mxfp4" else 16
    b = (gu + dn) // 2 + (gu + dn) // B
    if cfg.fmt == "nvfp4":
        b += 8
    return b, gu // 2 + gu // B + (4 if cfg.fmt == "nvfp4" else 0)


def is_prefill(cfg):
    return "prefill" in cfg.name


def uses_tensor_cores(cfg, variant=0):
    """The library's kernel choice for these weights: the bench gives MXFP4 weights their
    re-laid scale atoms, so MXFP4 runs on the tensor cores unless variant 1 forces the GEMV."""
    if variant:
        return variant == 2
    return cfg.fmt == "mxfp4"


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


# ------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
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
# our implementation
# ------------------------------------------------------------------------------------
def build_layer(cfg, copies, device):
    import torch
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from helpers import device_weights
    import dataclasses
    weights = [device_weights(cfg, device=device)]
    for _ in range(copies - 1):
        w0 = weights[0]
        # an independent copy of every device tensor (codes, scales, codebooks, CSR)
        weights.append(dataclasses.replace(w0, **{f.name: getattr(w0, f.name).clone()
                                                  for f in dataclasses.fields(w0)
                                                  if isinstance(getattr(w0, f.name), torch.Tensor)}))
    x_bits = D.activations_bf16(cfg.seed, cfg.T, cfg.H)
    wr = D.router_weights(cfg.seed, cfg.E, cfg.H)
    bias = D.zipf_bias(cfg.seed, cfg.E) if cfg.zipf_bias else None
    x = torch.from_numpy(x_bits.view(np.int16)).to(device).view(torch.bfloat16)
    wr_t = torch.from_numpy(wr).to(device)
    bias_t = None if bias is None else torch.from_numpy(bias).to(device)
    return weights, x, wr_t, bias_t, x_bits


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


def run_ours(args, cfg, rank, world):
    import torch
    import torch.distributed as dist
    from fp4_block_scaled_moe_b200 import api
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(device)
    per, _ = per_expert_bytes(cfg)
    bank_bytes = per * cfg.E
    copies = max(2, int(np.ceil(2 * L2_BYTES / bank_bytes)) + 1) if bank_bytes < 4 * L2_BYTES else 1
    weights, x, wr, bias, x_bits = build_layer(cfg, copies, device)
    from fp4_block_scaled_moe_b200 import prepare_mma_scales
    for w in weights:
        w.kernel_variant = args.variant
        if cfg.fmt == "mxfp4":
            prepare_mma_scales(w)        # one-time weight preparation, outside the timed region
    structs = [w.c_struct() for w in weights]
    T, k = cfg.T, cfg.k
    ws_bytes = api.moe_fp4_workspace_size(weights[0], T, k)
    ws = api.alloc_workspace(ws_bytes, device)
    y = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=device)
    route = {"counts": torch.empty(cfg.E, dtype=torch.int32, device=device)}
    stream = torch.cuda.Stream(device)

    def step(i):
        api.moe_fp4_forward(weights[i % copies], x, wr, bias, k, workspace=ws, y=y, _struct=structs[i % copies],
                            route_out=route if i == 0 else None)

    with torch.cuda.stream(stream):
        step(0)
    torch.cuda.synchronize()
    counts = route["counts"].cpu().numpy()
    extra_gu = extra_all = None
    if cfg.fmt == "cb4":
        extra_gu, extra_all = cb4_extra_bytes(weights[0])
    work_step, _ = work_per_step(cfg, counts, extra=extra_all)
    bytes_step = algorithmic_bytes(cfg, counts, extra=extra_all)
    # one CUDA graph per weight copy (kernel launches replayed without host overhead)
    graphs = []
    for c in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            step(c)                       # warm the launch path for this copy
            torch.cuda.synchronize()
            n0 = api.fp4_launch_count()
            with torch.cuda.graph(g, stream=stream):
                step(c)
            launches_per_step = api.fp4_launch_count() - n0
        graphs.append(g)
    torch.cuda.synchronize()
    for i in range(args.warmup):
        with torch.cuda.stream(stream):
            graphs[i % copies].replay()
    torch.cuda.synchronize()
    api.fp4_workspace_kernel_stats(ws, reset=True)
    clk = ClockSampler(device.index if device.index is not None else 0)
    if not args.no_clocks:
        clk.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        with torch.cuda.stream(stream):
            graphs[i % copies].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = e0.elapsed_time(e1)
    clocks = clk.stop() if not args.no_clocks else None

    kern = api.fp4_workspace_kernel_stats(ws)

    # end to end through the C ABI with host buffers: H2D of x, layer, D2H of y each step
    x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((T, cfg.H), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    for i in range(3):
        with torch.cuda.stream(stream):
            x_dev.copy_(x_host, non_blocking=True)
            api.moe_fp4_forward(weights[i % copies], x_dev, wr, bias, k, workspace=ws, y=y,
                                _struct=structs[i % copies])
            y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for i in range(args.steps):
        with torch.cuda.stream(stream):
            x_dev.copy_(x_host, non_blocking=True)
            api.moe_fp4_forward(weights[i % copies], x_dev, wr, bias, k, workspace=ws, y=y,
                                _struct=structs[i % copies])
            y_host.copy_(y, non_blocking=True)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a0.elapsed_time(a1)
    status = api.fp4_workspace_status(ws)

    gu_ms = kern["gate_up_ns"] / max(kern["gate_up_launches"], 1) / 1e6
    dn_ms = kern["down_ns"] / max(kern["down_launches"], 1) / 1e6
    ms_total, e2e_ms, gu_ms, dn_ms = max_over_ranks([ms_total, e2e_ms, gu_ms, dn_ms], world, device)
    kern_ms = {"gate_up": gu_ms, "down": dn_ms, "launches": kern["gate_up_launches"]}
    return dict(ms_per_step=ms_total / args.steps, bytes_step=bytes_step, work_step=work_step, extra_gu=extra_gu,
                e2e_ms=e2e_ms / args.steps,
                kern=kern, kern_ms=kern_ms, clocks=clocks, copies=copies, counts=counts, status=status,
                h2d=T * cfg.H * 2, d2h=T * cfg.H * 2, launches_per_step=launches_per_step)


# ------------------------------------------------------------------------------------
# reference arm / CPU baseline: the oracle on a bounded sample
# ------------------------------------------------------------------------------------
def oracle_sample(cfg, n_tokens):
    """Quantise (untimed) and return a closure running the oracle layer on n_tokens tokens."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from helpers import LazyOracleBank
    from oracle import moe as M, routing as R
    x_bits = D.activations_bf16(cfg.seed, cfg.T, cfg.H)
    wr = D.router_weights(cfg.seed, cfg.E, cfg.H)
    bias = D.zipf_bias(cfg.seed, cfg.E) if cfg.zipf_bias else None
    xf = D.bf16_bits_to_f32(x_bits)
    tok = np.arange(n_tokens)
    bank = LazyOracleBank(cfg)
    lg = R.router_logits(xf[tok], wr, bias)
    ids = R.topk(lg, cfg.k)
    for e in np.unique(ids):
        bank.packed("gu", int(e))
        bank.packed("dn", int(e))
    counts = np.bincount(ids.reshape(-1), minlength=cfg.E)
    extra = None
    if cfg.fmt == "cb4":            # CSR bytes of the sampled experts, from the oracle's own fits
        extra = np.zeros(cfg.E, dtype=np.int64)
        for e in np.unique(ids):
            for which, rows in (("gu", 2 * cfg.I), ("dn", cfg.H)):
                extra[e] += 6 * int(bank.packed(which, int(e))["row_ptr"][-1]) + 4 * rows

    def run():
        M.moe_layer(xf[tok], wr, bias, cfg.k, bank, cfg.swiglu_limit)

    return run, work_per_step(cfg, counts, tokens=n_tokens, extra=extra)[0]


# DRAM bytes (read + write) per launch of the dominant kernel from one ncu capture of the
# current build (profiles/): the decode layer's gate_up kernel (tensor-core and GEMV
# variants), and the prefill
# gate_up bs_moe_kernel captured at a quarter of the experts and tokens and scaled by the
# four times as many work units of the full layer.  None when no capture matches.
NCU_TRAFFIC = {
    ("moe_mxfp4_decode_e64_h2048_i768_k8_t16", "decode_kernel<gate_up+swiglu>"): 100_664_576,
    ("moe_mxfp4_decode_e64_h2048_i768_k8_t16", "bs_moe_kernel<gate_up+swiglu>"): 101_671_424,
    ("moe_mxfp4_prefill_e256_h6144_i2048_k8_t8192", "bs_moe_kernel<gate_up+swiglu>"): 4 * 1_134_384_488,
}


def roofline(cfg, r, hbm_peak, peaks, tensor=False):
    """Dominant kernel: gate_up with the fused SwiGLU, timed per launch on the device.
    Prefill: algorithmic flops per launch 4 T k H I against the measured bf16 peak (the
    two-term E4M3 x E2M1 MMAs run at the FP8 rate, twice the MMA work of one bf16 pass,
    so the bf16 rate is their ceiling for these flops).
    Decode: algorithmic bytes per launch =
    codes + scales of the gate_up rows of every routed expert + the f16 activation rows
    read once per unit + h written; duration = its device time per launch in the timed region."""
    ms = r["kern_ms"]["gate_up"]
    if is_prefill(cfg):
        flops = 4 * cfg.T * cfg.k * cfg.H * cfg.I
        ach = flops / (ms * 1e-3) / 1e12 if ms > 0 else None
        peak = peaks.get("bf16_tflops", 1590.0)
        return {"kernel": "bs_moe_kernel<gate_up+swiglu>", "bound": "tensor", "achieved": ach, "peak": peak,
                "unit": "TFLOP/s", "frac": (ach / peak) if ach else None,
                "traffic": NCU_TRAFFIC.get((cfg.name, "bs_moe_kernel<gate_up+swiglu>")),
                "peak_source": ("MEASURED_PEAKS.json bf16_tflops, burst (of measured)" if "bf16_tflops" in peaks
                                else "fallback 1590 TFLOP/s bf16 (of fallback)"),
                "frac_of_sustained": (ach / peaks["bf16_tflops_sustained"]) if ach and "bf16_tflops_sustained" in peaks
                else None,
                "flops_per_launch": int(flops), "ms_per_launch": ms, "down_ms_per_launch": r["kern_ms"]["down"],
                "timer": "device globaltimer per launch, accumulated in the workspace over the timed steps"}
    _, gu_per_expert = per_expert_bytes(cfg)
    d = int(np.count_nonzero(r["counts"]))
    P = cfg.T * cfg.k
    alg = d * gu_per_expert + cfg.T * cfg.H * 2 + P * cfg.I * 2
    if r.get("extra_gu") is not None:
        alg += int(np.sum(r["extra_gu"][r["counts"] > 0]))
    ach = alg / (ms * 1e-3) / 1e9 if ms > 0 else None
    kname = "bs_moe_kernel<gate_up+swiglu>" if tensor else "decode_kernel<gate_up+swiglu>"
    return {"kernel": kname, "bound": "hbm", "achieved": ach, "peak": hbm_peak,
            "unit": "GB/s", "frac": (ach / hbm_peak) if ach else None, "traffic": NCU_TRAFFIC.get((cfg.name, kname)),
            "peak_source": "MEASURED_PEAKS.json hbm_gbs (of measured)" if "hbm_gbs" in peaks else "fallback",
            "bytes_per_launch": int(alg), "ms_per_launch": ms, "down_ms_per_launch": r["kern_ms"]["down"],
            "timer": "device globaltimer per launch, accumulated in the workspace over the timed steps"}


def cpu_baseline(cfg, budget_s=20.0):
    """The float64 oracle timed on this host's cores on a bounded sample of the same
    workload: the layer for the first tokens (all their routed experts), repeated until
    about budget_s of CPU time; value in the metric's unit (algorithmic GB/s)."""
    n_tok = 1 if is_prefill(cfg) else min(cfg.T, 4)
    run, sample_work = oracle_sample(cfg, n_tok)
    run()                                            # warm (dequantise caches, BLAS threads)
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        dt = time.perf_counter() - t0
        if dt > budget_s or reps >= 50:
            break
    per = dt / reps
    return {"value": sample_work / per, "unit": work_per_step(cfg, np.ones(1))[1], "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"first {n_tok} of {cfg.T} tokens with all their routed experts, float64 numpy, "
                      f"{reps} repetitions in {dt:.1f} s", "ms_per_sample": per * 1e3}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def main():
    args = parse()
    cfg = C.FULL.get(args.config) or C.PROFILE[args.config]
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    metric = "FP4 MoE layer: decode HBM GB/s (% of peak); prefill TFLOP/s; tokens/s"
    workload = cfg.name
    if args.impl == "reference":
        if rank != 0:
            return
        n_tok = 1
        run, sample_work = oracle_sample(cfg, n_tok)
        unit = work_per_step(cfg, np.ones(1))[1]
        for _ in range(args.warmup):
            run()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            run()
        dt = (time.perf_counter() - t0) / args.steps
        v = sample_work / dt
        line = {"impl": "reference", "metric": metric, "value": v, "unit": unit, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": workload, "sample": f"{n_tok} token(s) of {cfg.T}, all their experts"},
                "cpu_baseline": {"value": v, "unit": unit, "cores": blas_threads(), "kind": "oracle",
                                 "sample": f"{n_tok} token(s) of {cfg.T}, float64 numpy oracle"},
                "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    r = run_ours(args, cfg, rank, world)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        pass
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    unit = work_per_step(cfg, r["counts"])[1]
    value = job_rate(r["work_step"], world, r["ms_per_step"])
    bank_mb = r["copies"] * per_expert_bytes(cfg)[0] * cfg.E / 1e6
    conf = {"workload": workload, "tokens": cfg.T, "experts": cfg.E, "hidden": cfg.H, "inter": cfg.I,
            "top_k": cfg.k, "format": cfg.fmt, "parallelism": f"replicas{world}",
            "l2": (f"weights rotate over {r['copies']} copies ({bank_mb:.0f} MB) > L2" if r["copies"] > 1
                   else f"weights {bank_mb:.0f} MB > L2, one copy"),
            "distinct_experts": int(np.count_nonzero(r["counts"])),
            "expert_kernels": "tensor-core block-scaled" if uses_tensor_cores(cfg, args.variant) else "CUDA-core grouped GEMV",
            "bytes_per_step": int(r["bytes_step"])}
    if is_prefill(cfg):
        conf["tokens_per_s"] = cfg.T * world / (r["ms_per_step"] * 1e-3)
        conf["pct_of_bf16_measured_peak"] = 100 * value / world / peaks.get("bf16_tflops", 1590.0)
        conf["pct_of_fp4_dense_nominal_9000"] = 100 * value / world / 9000.0
    else:
        conf["pct_of_hbm_peak"] = 100 * value / world / hbm_peak
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": ("e4m3x2xe2m1->f32" if uses_tensor_cores(cfg, args.variant)
                  else ("f16(codebook)xf16->f32" if cfg.fmt == "cb4" else "f16xe2m1->f32")),
        "data": "synthetic",
        "config": conf,
        "e2e": {"value": job_rate(r["work_step"], world, r["e2e_ms"]), "unit": unit,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches_per_step"] * args.steps,
        "roofline": roofline(cfg, r, hbm_peak, peaks, uses_tensor_cores(cfg, args.variant)),
        "clocks": r["clocks"],
        "device_status": r["status"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Build the in-tree shared libraries for sm_100a with nvcc.

    python -m fp4_block_scaled_moe_b200.build          # builds what is out of date
    python -m fp4_block_scaled_moe_b200.build --force

Outputs (git-ignored, shipped with the source tree):
  fp4_block_scaled_moe_b200/libfp4moe.so   the C-ABI library (include/fp4moe.h)
  synth/libfp4synth.so                     the device-side input generator
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr"]

TARGETS = {
    os.path.join(PKG, "libfp4moe.so"): {
        "srcs": ["api.cu", "pack.cu", "route.cu", "decode.cu", "bs_moe.cu", "nv_moe.cu", "cb4.cu", "v2a.cu", "dense16.cu", "moe.cu",
                 "no_alloc.cu"],
        "dir": os.path.join(PKG, "csrc"),
        "inc": [os.path.join(ROOT, "include"), os.path.join(PKG, "csrc")],
    },
    os.path.join(ROOT, "synth", "libfp4synth.so"): {
        "srcs": ["synth_gen.cu"],
        "dir": os.path.join(ROOT, "synth", "csrc"),
        "inc": [],
    },
}


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps(t):
    spec = TARGETS[t]
    files = [os.path.join(spec["dir"], s) for s in spec["srcs"]]
    for d in [spec["dir"]] + spec["inc"]:
        for f in os.listdir(d):
            if f.endswith((".cuh", ".h")):
                files.append(os.path.join(d, f))
    return files


def _stale(t) -> bool:
    if not os.path.exists(t):
        return True
    mt = os.path.getmtime(t)
    return any(os.path.getmtime(f) > mt for f in _deps(t))


def _compile(src, obj, inc, verbose):
    cmd = [nvcc()] + ARCH + NVCC_FLAGS + [f"-I{i}" for i in inc] + ["-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return r.stderr


def build_target(t, verbose=False):
    spec = TARGETS[t]
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    with cf.ThreadPoolExecutor(max_workers=min(8, len(spec["srcs"]))) as ex:
        futs = []
        for s in spec["srcs"]:
            obj = os.path.join(BUILD, os.path.basename(t) + "." + s + ".o")
            objs.append(obj)
            futs.append(ex.submit(_compile, os.path.join(spec["dir"], s), obj, spec["inc"], verbose))
        for f in futs:
            msg = f.result()
            if verbose and msg:
                sys.stderr.write(msg)
    tmp = t + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed for {t}:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, t)


HOST_TARGETS = {
    os.path.join(ROOT, "synth", "libfp4synth_host.so"): os.path.join(ROOT, "synth", "csrc", "synth_host.c"),
}


def build_host(t, src):
    tmp = t + ".tmp"
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", src, "-o", tmp,
           "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"gcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, t)


def build(force: bool = False, verbose: bool = False):
    for t in TARGETS:
        if force or _stale(t):
            build_target(t, verbose)
    for t, src in HOST_TARGETS.items():
        if force or not os.path.exists(t) or os.path.getmtime(src) > os.path.getmtime(t):
            build_host(t, src)
    return list(TARGETS) + list(HOST_TARGETS)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register / smem usage")
    args = ap.parse_args()
    for t in build(args.force, args.verbose):
        print(t)

"""Build the in-tree shared libraries with nvcc for sm_100a.

    python long_context_layer_b200/build.py [--force]

(Run it by path: importing the package loads the library this script builds.)

Produces long_context_layer_b200/libdelta_attn.so (the C ABI of include/delta_attn.h),
synth/libsynth_fill.so (the device-side input generator used by tests and the benchmark) and
synth/libsynth_host.so (the same generator on the host, for fast oracle inputs).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared"]

TARGETS = [
    (os.path.join(ROOT, "long_context_layer_b200", "csrc", "delta_attn.cu"),
     os.path.join(ROOT, "long_context_layer_b200", "libdelta_attn.so"),
     ["-I" + os.path.join(ROOT, "include")]),
    (os.path.join(ROOT, "synth", "csrc", "synth_fill.cu"),
     os.path.join(ROOT, "synth", "libsynth_fill.so"), []),
]
# host (CPU) libraries built with gcc: the input generator's host copy
HOST_TARGETS = [
    (os.path.join(ROOT, "synth", "csrc", "synth_host.c"), os.path.join(ROOT, "synth", "libsynth_host.so")),
]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def build(force: bool = False, verbose: bool = False) -> list:
    built = []
    for src, out, extra in TARGETS:
        csrc = os.path.dirname(src)
        deps = [os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh", ".h"))]
        deps += [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]
        if not force and os.path.exists(out) and os.path.getmtime(out) >= max(os.path.getmtime(d) for d in deps):
            continue
        cmd = [nvcc()] + ARCH + COMMON + extra + [src, "-o", out]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        built.append(out)
    for src, out in HOST_TARGETS:
        if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
            continue
        cmd = ["gcc", "-O3", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", src, "-o", out]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        built.append(out)
    return built


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)

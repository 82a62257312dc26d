"""Builds libple.so (the layer) and ple_inputs/libple_synth.so (the synthetic
table filler) in-tree with nvcc for sm_100a. No GPU is needed to build.

    python -m gram_embedding_lookup_b200.build
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
          "-Xptxas", "-v"]

LIBPLE_SOURCES = ["ple_api.cu", "ple_kernels.cu", "ple_gemm.cu", "ple_decode.cu", "ple_mtp.cu", "ple_static.cu"]
LIBPLE = os.path.join(PKG, "libple.so")
LIBSYNTH = os.path.join(ROOT, "ple_inputs", "libple_synth.so")
SYNTH_SOURCES = [os.path.join(ROOT, "ple_inputs", "csrc", "ple_synth.cu")]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _needs_build(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    deps = list(sources)
    for d in (CSRC, INCLUDE):
        deps += [os.path.join(d, f) for f in os.listdir(d)]
    return any(os.path.getmtime(s) > t for s in deps if os.path.isfile(s))


def _run(cmd, log):
    res = subprocess.run(cmd, capture_output=True, text=True)
    if log is not None:
        with open(log, "w") as f:
            f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed ({res.returncode}): {' '.join(cmd)}")
    return res


def build(force: bool = False, ptxas_log: str | None = None) -> None:
    nvcc = _nvcc()
    srcs = [os.path.join(CSRC, s) for s in LIBPLE_SOURCES]
    if force or _needs_build(LIBPLE, srcs):
        tmp = LIBPLE + ".tmp"
        _run([nvcc, *ARCH, *COMMON, "-I", INCLUDE, "-I", CSRC, *srcs, "-o", tmp], ptxas_log)
        os.replace(tmp, LIBPLE)
    if force or _needs_build(LIBSYNTH, SYNTH_SOURCES):
        tmp = LIBSYNTH + ".tmp"
        _run([nvcc, *ARCH, *[f for f in COMMON if f not in ("-Xptxas", "-v")], *SYNTH_SOURCES, "-o", tmp], None)
        os.replace(tmp, LIBSYNTH)


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_log=None)
    print("built", LIBPLE, LIBSYNTH)

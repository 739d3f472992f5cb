"""In-tree build of the native libraries.

* ``libpi.so``            — the C-ABI library (CUDA kernels for sm_100a + host
                            entry points), from ``csrc/*.cu``.
* ``synth/libpi_synth_dev.so``  — the device side of the input generator.
* ``synth/libpi_synth_host.so`` — the host side of the input generator (gcc).

Everything is compiled for ``sm_100a`` only (``-gencode
arch=compute_100a,code=sm_100a``); nvcc cross-compiles without a GPU.
Rebuilds when a source or header is newer than its output.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
SYNTH = os.path.join(PKG, "synth")

LIBPI = os.path.join(PKG, "libpi.so")
SYNTH_DEV = os.path.join(SYNTH, "libpi_synth_dev.so")
SYNTH_HOST = os.path.join(SYNTH, "libpi_synth_host.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
              "--expt-relaxed-constexpr", "-Xptxas=-warn-spills"]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build_synth(force: bool = False, verbose: bool = False) -> None:
    deps = [os.path.join(SYNTH, "rng.h"), os.path.join(SYNTH, "synth_host.c")]
    if force or _stale(SYNTH_HOST, deps):
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                        "-ffp-contract=off", "-o", SYNTH_HOST,
                        os.path.join(SYNTH, "synth_host.c"), "-lm"], check=True)
    deps = [os.path.join(SYNTH, "rng.h"), os.path.join(SYNTH, "synth_dev.cu")]
    if force or _stale(SYNTH_DEV, deps):
        subprocess.run([_nvcc(), *ARCH, "-O3", "-fmad=false", "-Xcompiler", "-fPIC",
                        "-shared", "-o", SYNTH_DEV, os.path.join(SYNTH, "synth_dev.cu")],
                       check=True)


def build_libpi(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
                out: str | None = None) -> str | None:
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    if not srcs:
        return None
    out = out or LIBPI
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    if force or _stale(out, deps):
        cmd = [_nvcc(), *ARCH, *NVCC_FLAGS, f"-I{INCLUDE}", f"-I{CSRC}", *(extra or []),
               "-o", out, *srcs]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
    return out


def build(force: bool = False, verbose: bool = False) -> None:
    build_synth(force, verbose)
    build_libpi(force, verbose)


if __name__ == "__main__":
    import sys
    build(force="--force" in sys.argv, verbose=True)

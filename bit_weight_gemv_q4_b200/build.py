"""Build the native libraries of the package in-tree.

* ``libq4gemv.so``  -- the C-ABI product library: the host packer and the
  sm_100a CUDA kernels (``csrc/pack.cpp``, ``csrc/q4gemv.cu``).
* ``libq4synth.so`` -- the seeded synthetic-input generator (``csrc/synth.cu``,
  one definition in ``csrc/synth_core.h`` compiled for host and device,
  without floating-point contraction so both give identical bits).

Run ``python -m bit_weight_gemv_q4_b200.build`` or call :func:`build_all`.
A library is rebuilt only when one of its sources is newer than it.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

GEMV_LIB = os.path.join(HERE, "libq4gemv.so")
SYNTH_LIB = os.path.join(HERE, "libq4synth.so")

GEMV_SOURCES = [os.path.join(CSRC, "q4gemv.cu"), os.path.join(CSRC, "pack.cpp"), os.path.join(CSRC, "quantize.cu"),
                os.path.join(CSRC, "spec.cu")]
GEMV_DEPS = GEMV_SOURCES + [os.path.join(INCLUDE, "q4gemv.h"), os.path.join(CSRC, "q4gemv_kernels.cuh"),
                            os.path.join(CSRC, "q4stack_kernel.cuh"), os.path.join(CSRC, "q4chain_kernel.cuh"),
                            os.path.join(CSRC, "q4nvfp4_kernel.cuh"), os.path.join(CSRC, "q4spec_kernel.cuh"),
                            os.path.join(CSRC, "q4wide_kernel.cuh"), os.path.join(CSRC, "q4chainp_kernel.cuh")]
SYNTH_SOURCES = [os.path.join(CSRC, "synth.cu")]
SYNTH_DEPS = SYNTH_SOURCES + [os.path.join(CSRC, "synth_core.h")]

NVCC_ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libq4gemv.so")


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.exists(d) and os.path.getmtime(d) > t for d in deps)


def _run(cmd: list[str]) -> None:
    proc = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if proc.returncode != 0:
        raise RuntimeError("build failed:\n" + " ".join(cmd) + "\n" + proc.stdout)


def build_synth(force: bool = False) -> str:
    if force or _stale(SYNTH_LIB, SYNTH_DEPS):
        tmp = SYNTH_LIB + ".tmp"
        _run([_nvcc(), *NVCC_ARCH, "-O3", "-std=c++17", "-shared", "-fmad=false",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-ffp-contract=off", "-Xcompiler", "-fopenmp",
              "-Xcompiler", "-fvisibility=hidden", "-cudart", "static", *SYNTH_SOURCES, "-o", tmp, "-lgomp"])
        os.replace(tmp, SYNTH_LIB)
    return SYNTH_LIB


def build_gemv(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or _stale(GEMV_LIB, GEMV_DEPS):
        tmp = GEMV_LIB + ".tmp"
        cmd = [_nvcc(), *NVCC_ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
               "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-Xcompiler", "-fopenmp",
               "-I", INCLUDE, "-cudart", "static", *GEMV_SOURCES, "-o", tmp, "-lgomp"]
        if verbose_ptxas:
            cmd[1:1] = ["-Xptxas", "-v"]
        _run(cmd)
        os.replace(tmp, GEMV_LIB)
    return GEMV_LIB


def build_all(force: bool = False) -> None:
    build_synth(force)
    build_gemv(force)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
    print("built", GEMV_LIB, SYNTH_LIB)

"""CPU oracle of the group-quantised weight x activation product -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
has no CPU fallback.  It shares no code with the CUDA library: the two meet only
at the canonical input layout written by the seeded generator.

``gemv`` follows the plain definition (dequantise each weight to fp32 as
scale * integer, which is exact, and accumulate weight * activation in fp64):

    y[m, n] = sum_k s[n, k // 32] * q[n, k] * x[m, k]
    B[m, n] = sum_k |s[n, k // 32] * q[n, k] * x[m, k]|

Sources: the weight stream of single-user decode is 4-bit weights with 16-bit
activations (jdon.com "Two RTX 3090s, 105 tok/s", sections "27 billion
parameters into 24 GB" and "Schools of quantisation"), with 8-bit tensors for
the sensitive projections and the output head (bs178.com llamAmpere post,
"Why it is this fast", part two).  Group size 32, one fp16 scale per group and
the symmetric [-8, 7] / [-127, 127] ranges are the plain reading the pages leave
open; ``layout.py`` decodes the kernel-native packed layout from its written
specification, and ``quantize.py`` is the offline quantiser (bf16 weights to
codes and fp16 scales) with every rounding step fixed.  ``chain.py`` holds the
steps between the products of a dependent decode chain, ``nvfp4.py`` the NVFP4
weight format, and ``spec.py`` the MTP draft / verify step (rejection sampling
over the draft head's mapped vocabulary).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "oracle.c")

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c (plain C, OpenMP) into liboracle.so next to it."""
    if force or not os.path.exists(LIB) or os.path.getmtime(SRC) > os.path.getmtime(LIB):
        tmp = LIB + ".tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", SRC, "-o", tmp, "-lm"]
        proc = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
        if proc.returncode != 0:
            raise RuntimeError("oracle build failed:\n" + proc.stdout)
        os.replace(tmp, LIB)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        L.oracle_f16_value.argtypes = [ctypes.c_uint16]
        L.oracle_f16_value.restype = ctypes.c_double
        L.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_value.restype = ctypes.c_double
        L.oracle_q4_value.argtypes = [vp, i64]
        L.oracle_q4_value.restype = ctypes.c_int
        L.oracle_gemv.argtypes = [ctypes.c_int, vp, vp, i64, i64, vp, ctypes.c_int, vp, vp]
        L.oracle_gemv.restype = ctypes.c_int
        L.oracle_dequantize.argtypes = [ctypes.c_int, vp, vp, i64, i64, vp]
        L.oracle_dequantize.restype = ctypes.c_int
        L.oracle_threads.argtypes = []
        L.oracle_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


_WIDE_RANGE = {5: 16, 6: 32}  # q5 / q6: int8 codes in [-r, r - 1]


def _narrow(bits: int, q: np.ndarray) -> int:
    """q5 and q6 codes are int8 [N][K] like q8's, in a narrower range; the
    definition (s * q * x summed) is the same, so they take the q8 routine."""
    if bits in _WIDE_RANGE:
        r = _WIDE_RANGE[bits]
        qa = np.asarray(q)
        if qa.size and (qa.min() < -r or qa.max() > r - 1):
            raise ValueError(f"q{bits} codes must lie in [{-r}, {r - 1}]")
        return 8
    return bits


def gemv(bits: int, q: np.ndarray, s: np.ndarray, x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(y, B) in fp64, each [M][N], for canonical q ([N][K/2] uint8 or [N][K] int8),
    fp16-bit scales s [N][K/32] and bf16-bit activations x [M][K]."""
    bits = _narrow(bits, q)
    x = _c(np.atleast_2d(x), np.uint16)
    M, K = x.shape
    N = q.shape[0]
    q = _c(q, np.uint8 if bits == 4 else np.int8)
    s = _c(s, np.uint16)
    if bits == 4 and q.shape != (N, K // 2):
        raise ValueError("q4 weights must be [N][K/2]")
    if bits == 8 and q.shape != (N, K):
        raise ValueError("q8 weights must be [N][K]")
    if s.shape != (N, K // 32):
        raise ValueError("scales must be [N][K/32]")
    y = np.empty((M, N), dtype=np.float64)
    B = np.empty((M, N), dtype=np.float64)
    rc = lib().oracle_gemv(bits, q.ctypes.data, s.ctypes.data, N, K, x.ctypes.data, M, y.ctypes.data, B.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_gemv: bad arguments")
    return y, B


def dequantize(bits: int, q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Dense W[n][k] = s[n][k/32] * q[n][k] as fp64."""
    bits = _narrow(bits, q)
    N = q.shape[0]
    K = s.shape[1] * 32
    q = _c(q, np.uint8 if bits == 4 else np.int8)
    s = _c(s, np.uint16)
    W = np.empty((N, K), dtype=np.float64)
    if lib().oracle_dequantize(bits, q.ctypes.data, s.ctypes.data, N, K, W.ctypes.data) != 0:
        raise ValueError("oracle_dequantize: bad arguments")
    return W


def f16_value(h: int) -> float:
    return lib().oracle_f16_value(int(h) & 0xFFFF)


def bf16_value(b: int) -> float:
    return lib().oracle_bf16_value(int(b) & 0xFFFF)


def q4_value(row: np.ndarray, k: int) -> int:
    row = _c(row, np.uint8)
    return lib().oracle_q4_value(row.ctypes.data, k)


def bf16_array(x: np.ndarray) -> np.ndarray:
    """Decode an array of bf16 bits to fp64 through the oracle's own decoder."""
    flat = np.asarray(x, dtype=np.uint16).ravel()
    out = np.fromiter((lib().oracle_bf16_value(int(v)) for v in flat), dtype=np.float64, count=flat.size)
    return out.reshape(np.shape(x))


def threads() -> int:
    return lib().oracle_threads()


def within_tolerance(y: np.ndarray, y_ref: np.ndarray, B: np.ndarray, rel: float = 1e-3, abs_: float = 1e-6):
    """Element-wise |y - y_ref| <= rel * B + abs_ (the pass criterion of the product)."""
    err = np.abs(np.asarray(y, dtype=np.float64) - y_ref)
    bound = rel * B + abs_
    return err <= bound, err, bound

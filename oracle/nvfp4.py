"""CPU oracle of the NVFP4 weight format -- TEST INFRASTRUCTURE (see __init__.py).

The pages name NVFP4 as the 4-bit format Blackwell engines run
(ai-coding.wiselychen.com guide, section "RTX 5090 32GB": SGLang / vLLM +
NVFP4) without defining it; the published definition is used: blocks of 16
consecutive values along K, each value an FP4 E2M1 number (1 sign, 2
exponent, 1 mantissa bit, exponent bias 1, no inf / NaN), one FP8 E4M3 scale
per block (1 sign, 4 exponent, 3 mantissa bits, bias 7, subnormals, no inf,
S.1111.111 = NaN), and one fp32 scale per tensor:

    w[n][k] = t * e4m3(s[n][k // 16]) * e2m1(c[n][k])
    y[m][n] = sum_k w[n][k] * x[m][k]              (fp64)

Canonical layout: codes uint8 [N][K/2] (element k in byte k/2, low nibble for
even k), block scales uint8 [N][K/16] (E4M3 bits), t a float32.
"""
from __future__ import annotations

import numpy as np


def e2m1_value(code: int) -> float:
    """The E2M1 number of a 4-bit code, from the bit fields."""
    sign = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:  # subnormal: m * 2^(1 - bias) * 0.5
        return sign * m * 0.5
    return sign * (1.0 + 0.5 * m) * 2.0 ** (e - 1)


def e4m3_value(byte: int) -> float:
    """The E4M3 number of a byte, from the bit fields (NaN for S.1111.111)."""
    sign = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 7
    if e == 0xF and m == 7:
        return float("nan")
    if e == 0:
        return sign * m / 8.0 * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E2M1 = np.array([e2m1_value(c) for c in range(16)])
E4M3 = np.array([e4m3_value(b) for b in range(256)])


def codes_to_ints(codes: np.ndarray, K: int) -> np.ndarray:
    """Canonical code bytes [N][K/2] -> 4-bit codes [N][K]."""
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty((c.shape[0], K), dtype=np.uint8)
    out[:, 0::2] = c & 0xF
    out[:, 1::2] = c >> 4
    return out


def dequantize(codes: np.ndarray, scales: np.ndarray, t: float, K: int) -> np.ndarray:
    """Dense fp64 weights [N][K]."""
    c = codes_to_ints(codes, K)
    s = E4M3[np.asarray(scales, dtype=np.uint8)]  # [N][K/16]
    return np.float64(np.float32(t)) * s.repeat(16, axis=1) * E2M1[c]


def gemv(codes: np.ndarray, scales: np.ndarray, t: float, x_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(y fp64 [M][N], sum_k |w x| [M][N]) for bf16 activation bits x [M][K]."""
    x = (np.asarray(x_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    K = x.shape[1]
    w = dequantize(codes, scales, t, K)
    return x @ w.T, np.abs(x) @ np.abs(w).T

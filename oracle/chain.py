"""CPU oracle of a dependent decode chain -- TEST INFRASTRUCTURE (see __init__.py).

The products of one decode layer depend on each other through the steps
that sit between them: the residual stream h is updated with a product's
output, normalised, and rounded to bf16 to become the next product's
activations; the fused gate|up output goes through SwiGLU into the down
projection.  The pages name the layer structure (64 layers, 16 gated
attention and 48 Gated DeltaNet: ai-coding.wiselychen.com guide, section
"Before deploying: weights, KV cache, memory bandwidth") but define neither
step, so the plain textbook forms are used, in fp64:

  residual + RMSNorm:  h <- h + y (or h <- y, the step's first);
                       x = bf16( h / sqrt(mean_k h_k^2 + eps) * gamma ),  eps = 1e-6
  SwiGLU:              x = bf16( silu(g) * u ),  silu(z) = z / (1 + e^-z),
                       g = y[:, :N], u = y[:, N:2N] of the fused gate|up output
  product:             y = oracle.gemv(codes, scales, x)

bf16 rounding is to nearest, ties to even, as the library's conversion.
"""
from __future__ import annotations

import math

import numpy as np

import oracle

EPS = 1e-6


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bits, round to nearest even (via the exact fp32 value)."""
    a = np.asarray(a, dtype=np.float64)
    f = a.astype(np.float32)  # fp64 -> fp32 is round to nearest even
    u = f.view(np.uint32).astype(np.uint64)
    # fp32 -> bf16, nearest even, from the fp32 bits; a double rounding only
    # matters when the fp64 value lies within 2^-24 relative of a bf16 tie
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def bf16_exact(a: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bits, round to nearest even, in one step (exact arithmetic
    on the fp64 value; no intermediate fp32)."""
    a = np.asarray(a, dtype=np.float64)
    out = np.zeros(a.shape, dtype=np.uint16)
    for idx, v in np.ndenumerate(a):
        if v == 0.0 or not math.isfinite(v):
            out[idx] = bf16_bits(np.array([v]))[0]
            continue
        m, e = math.frexp(abs(v))  # v = m * 2^e, m in [0.5, 1)
        e_min = -125  # smallest normal bf16 is 2^-126 = 0.5 * 2^-125
        scale = 2.0 ** (8 - max(e, e_min))  # units of the last bf16 mantissa bit
        t = abs(v) * scale
        n = math.floor(t)
        rem = t - n
        if rem > 0.5 or (rem == 0.5 and n % 2 == 1):
            n += 1
        r = math.copysign(n / scale, v)
        out[idx] = bf16_bits(np.array([r]))[0]
    return out


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def silu(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def residual_rmsnorm(h: np.ndarray | None, y: np.ndarray | None, gamma: np.ndarray | None, eps: float = EPS):
    """h [M][N] or None (the step's first: h <- y), y [M][N] or None, gamma
    [N] or None (= 1) -> (h', z): the updated residual stream and the
    normalised values before the bf16 rounding (fp64)."""
    if h is None:
        h2 = np.array(y, dtype=np.float64)
    else:
        h2 = np.array(h, dtype=np.float64) + (0.0 if y is None else np.asarray(y, dtype=np.float64))
    rms = np.sqrt(np.mean(h2 * h2, axis=1, keepdims=True) + eps)
    z = h2 / rms
    if gamma is not None:
        z = z * np.asarray(gamma, dtype=np.float64)[None, :]
    return h2, z


def swiglu(y_gu: np.ndarray, N: int) -> np.ndarray:
    """y_gu [M][2N] (gate then up) -> z = silu(g) * u [M][N] before the bf16 rounding."""
    y_gu = np.asarray(y_gu, dtype=np.float64)
    return silu(y_gu[:, :N]) * y_gu[:, N:2 * N]


def near_bf16_tie(z: np.ndarray, rel: float) -> np.ndarray:
    """True where z lies within rel * |z| of a point half-way between two bf16
    values: there a faithful fp32 computation may round either way."""
    z = np.asarray(z, dtype=np.float64)
    a = np.abs(z)
    out = np.zeros(z.shape, dtype=bool)
    nz = a > 0
    m, e = np.frexp(a[nz])  # a = m 2^e, m in [0.5, 1)
    e = np.maximum(e, -125)
    t = a[nz] * np.ldexp(1.0, 8 - e)  # in units of the last bf16 bit
    frac = t - np.floor(t)
    out[nz] = np.abs(frac - 0.5) <= rel * t
    return out


def product(bits: int, q: np.ndarray, s: np.ndarray, x_bits: np.ndarray):
    """(y fp64 [M][N], sum |w x| [M][N]) of a product on bf16 activations."""
    return oracle.gemv(bits, q, s, x_bits)

"""CPU oracle of the offline quantiser -- TEST INFRASTRUCTURE (see __init__.py).

Round-to-nearest, group-32, symmetric (no zero point) quantisation of bf16
weights into the canonical code and scale layout, written as plain numpy,
step by step.  The pages say only that a quantiser's grouping,
scale computation and outlier handling matter (jdon.com "Two RTX 3090s, 105
tok/s", section "Schools of quantisation") and name 4-bit and 8-bit formats
(bs178.com llamAmpere post, "Why it is this fast", part two); the recipe below
is the plain reading, with every rounding step fixed so that any faithful
implementation produces the same bits:

For each row n and group g (32 consecutive k), with w the group's values as
fp32 (exact from bf16):

  absmax mode (4 and 8 bit):  s32 = max|w| / qmax          qmax = 7 or 127
  signed mode (4 bit only):   s32 = w_m / (-8)             w_m = the value of largest
                                                           magnitude, first in k order
  s16 = fp16 round-to-nearest-even of s32, saturated to +-65504
  s   = s16 as fp32
  q   = 0 if s == 0, else clamp(nearest(w / s), lo, hi)    the integer nearest to the
                                                           exact quotient, ties to even;
                                                           [lo, hi] = [-7, 7] absmax q4,
                                                           [-8, 7] signed q4, [-127, 127] q8

The quotient is formed in fp64 here: w has an 8-bit and s an 11-bit
significand, so a quotient that is not exactly half-way between two integers
lies at least 2^-21 from that half-way point whenever it is above 1/2 in
magnitude, far beyond the fp64 rounding error (2^-45 at most), and an exact
half-way quotient is exactly representable: rint of the fp64 quotient is the
nearest integer of the exact one, ties to even.

Absmax mode never uses the code -8; signed mode maps the largest-magnitude
value to -8 exactly and so uses all sixteen codes.  The outputs are the
canonical layouts: q4 as uint8 [N][K/2] (element k in byte k/2, low nibble for
even k, two's complement), q8 as int8 [N][K], scales as fp16 bits [N][K/32].
"""
from __future__ import annotations

import numpy as np

ABSMAX = 0
SIGNED_MAX = 1

F16_MAX = np.float32(65504.0)


def bf16_to_f32(w_bits: np.ndarray) -> np.ndarray:
    return (np.asarray(w_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def group_scales(bits: int, mode: int, wf: np.ndarray) -> np.ndarray:
    """wf: float32 [N][G][32] -> fp16 scales [N][G] (as np.float16)."""
    if mode == ABSMAX:
        qmax = np.float32(7.0 if bits == 4 else 127.0)
        s32 = (np.abs(wf).max(axis=2) / qmax).astype(np.float32)
    elif mode == SIGNED_MAX and bits == 4:
        idx = np.abs(wf).argmax(axis=2)  # first maximum in k order
        wm = np.take_along_axis(wf, idx[..., None], axis=2)[..., 0]
        s32 = (wm / np.float32(-8.0)).astype(np.float32)
    else:
        raise ValueError("signed mode is defined for 4-bit codes only")
    with np.errstate(over="ignore"):
        s16 = s32.astype(np.float16)
    s16 = np.where(np.isinf(s16), np.sign(s32).astype(np.float16) * np.float16(65504.0), s16)
    return s16.astype(np.float16)


def code_range(bits: int, mode: int) -> tuple[int, int]:
    if bits == 8:
        return -127, 127
    return (-8, 7) if mode == SIGNED_MAX else (-7, 7)


def quantize_ints(bits: int, mode: int, w_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16 bits [N][K] -> (integer codes int32 [N][K], fp16 scale bits uint16 [N][K/32])."""
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    N, K = w_bits.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    wf = bf16_to_f32(w_bits).reshape(N, K // 32, 32)
    s16 = group_scales(bits, mode, wf)
    s = s16.astype(np.float32)[..., None]
    lo, hi = code_range(bits, mode)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = wf.astype(np.float64) / np.where(s == 0, np.float32(1.0), s).astype(np.float64)
    q = np.clip(np.rint(ratio), lo, hi)
    q = np.where(s == 0, 0, q).astype(np.int32)
    return q.reshape(N, K), s16.view(np.uint16)


def to_canonical(bits: int, q: np.ndarray) -> np.ndarray:
    """Integer codes [N][K] -> the canonical code layout."""
    if bits == 8:
        return q.astype(np.int8)
    nib = (q.astype(np.int64) & 0xF).astype(np.uint8)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def quantize(bits: int, mode: int, w_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16 bits [N][K] -> (canonical codes, fp16 scale bits [N][K/32])."""
    q, s = quantize_ints(bits, mode, w_bits)
    return to_canonical(bits, q), s

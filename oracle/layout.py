"""Decoder of the kernel-native packed layout -- TEST INFRASTRUCTURE.

Written from the layout's specification (the "Kernel-native packed layout"
block of include/q4gemv.h), in the opposite direction to the library's packer:
for every canonical element (n, k) it computes where the specification puts it
and reads it back.  It shares no code with the library.  The pages describe no
packed layout (the bs178.com llamAmpere post, "Why it is this fast", part one,
only says the fork "fixed the reads" and staged them with async copies); the
layout is this library's own design.
"""
from __future__ import annotations

import numpy as np

TILE_ROWS = 32


WIDE_SHIFT = {5: [-4, -3, -2, -1, 4, 5, 6, 7], 6: [-4, -2, 4, 6]}
WIDE_OFFSET = {5: 16, 6: 32}


def _geometry(bits: int, N: int, K: int):
    kc = 32 if bits == 8 else 64
    T = -(-N // TILE_ROWS)
    C = -(-K // kc)
    CB = {4: 1152, 5: 1408, 6: 1664, 8: 1088}[bits]
    return T, C, CB


def decode(bits: int, packed: np.ndarray, N: int, K: int) -> tuple[np.ndarray, np.ndarray]:
    """Integer weights q [N][K] (int64) and fp16 scale bits [N][K/32] from packed bytes."""
    T, C, CB = _geometry(bits, N, K)
    packed = np.asarray(packed, dtype=np.uint8)
    assert packed.size >= T * C * CB
    n = np.arange(N, dtype=np.int64)[:, None]
    k = np.arange(K, dtype=np.int64)[None, :]
    t = n // TILE_ROWS
    rr = n % TILE_ROWS
    h = rr // 16          # which 16-row half of the tile
    gi = rr % 8
    upper = (rr % 16) // 8  # 1 for the row R + 8 of the slot
    if bits in (4, 5, 6):
        c = k // 64
        kk = k % 64
        G = kk // 32
        within = kk % 32
        ti = within // 8
        e = (within % 8) // 4
        r4 = within % 4  # = 2*((i>>1)&1) + (i>>2)
        i = 4 * (r4 % 2) + 2 * (r4 // 2) + upper
        j = 2 * G + e
        off = (t * C + c) * CB + 512 * h + 16 * (4 * gi + ti) + 4 * j
        word = _word(packed, off)
        u = (word >> (4 * i).astype(np.uint32)) & 0xF
        if bits == 4:
            q = u.astype(np.int64) - 8
        else:
            lane = 4 * gi + ti
            reg, half = i % 4, i // 4
            sel = 2 * j + reg // 2 if bits == 5 else 2 * (j % 2) + reg // 2
            pos = 16 * half + np.asarray(WIDE_SHIFT[bits])[sel] + np.where(reg % 2 == 1, 8, 4)
            hoff = (t * C + c) * CB + (1024 + 8 * lane + 4 * h if bits == 5 else 1024 + 16 * lane + 8 * h + 4 * (j // 2))
            hi = (_word(packed, hoff) >> pos.astype(np.uint32)) & (1 if bits == 5 else 3)
            q = (u + 16 * hi).astype(np.int64) - WIDE_OFFSET[bits]
    else:
        c = k // 32
        within = k % 32
        ti = within // 8
        e = (within % 8) // 4
        r4 = within % 4  # = 2f + (b>>1)
        f = r4 // 2
        b = 2 * (r4 % 2) + upper
        j = 2 * e + f
        off = (t * C + c) * CB + 512 * h + 16 * (4 * gi + ti) + 4 * j
        word = _word(packed, off)
        u = (word >> (8 * b).astype(np.uint32)) & 0xFF
        q = u.astype(np.int64) - 128
    Gn = K // 32
    g = np.arange(Gn, dtype=np.int64)[None, :]
    if bits in (4, 5, 6):
        cs = g // 2
        slot = 4 * h + 2 * upper + (g % 2)
        sbase = {4: 1024, 5: 1280, 6: 1536}[bits]
        soff = (t * C + cs) * CB + sbase + 16 * gi + 2 * slot
    else:
        slot = 2 * h + upper
        soff = (t * C + g) * CB + 1024 + 8 * gi + 2 * slot
    s = packed[soff].astype(np.uint16) | (packed[soff + 1].astype(np.uint16) << 8)
    return q, s


def _word(packed: np.ndarray, off: np.ndarray) -> np.ndarray:
    b = [packed[off + m].astype(np.uint32) for m in range(4)]
    return b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24)


def padding_is_zero(bits: int, packed: np.ndarray, N: int, K: int) -> bool:
    """Rows >= N and groups >= K/32 of the padded tiles decode to q = 0, scale 0."""
    T, C, CB = _geometry(bits, N, K)
    Np = T * TILE_ROWS
    Kp = C * (32 if bits == 8 else 64)
    q, s = decode(bits, packed, Np, Kp)
    return bool(np.all(q[N:, :] == 0) and np.all(q[:, K:] == 0) and np.all(s[N:, :] == 0) and np.all(s[:, K // 32:] == 0))

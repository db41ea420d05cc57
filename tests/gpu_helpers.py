"""Shared helpers of the GPU tests: build inputs with the seeded generator, run
the library through its C-ABI binding, and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np

import oracle
from bit_weight_gemv_q4_b200 import synth


def torch():
    import torch as _t

    return _t


def host_inputs(bits, N, K, M, seed=0, tensor_id=1, act_id=None):
    q, s = synth.tensor(bits, seed, tensor_id, N, K)
    x = synth.activations(seed, synth.act_stream(tensor_id if act_id is None else act_id), M, K)
    return q, s, x


def to_device_packed(bits, q, s, N, K):
    import bit_weight_gemv_q4_b200 as q4

    t = torch()
    packed = q4.q4_pack_weights(bits, q, s, N, K)
    buf = t.empty(max(packed.size, 16), dtype=t.uint8, device="cuda")
    if packed.size:
        buf[: packed.size].copy_(t.from_numpy(packed))
    return buf


def to_device_x(x):
    t = torch()
    if x.size == 0:
        return t.empty(16, dtype=t.int16, device="cuda")
    return t.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda()


def workspace(bits, N, K, M):
    import bit_weight_gemv_q4_b200 as q4

    t = torch()
    return t.zeros(q4.q4_gemv_workspace_bytes(bits, N, K, M), dtype=t.uint8, device="cuda")


def run_gemv(bits, packed, N, K, x_dev, M, ws=None, guard=64):
    """Runs q4_gemv / q8_gemv into a y surrounded by NaN guard words; returns
    (y as numpy [M][N], guards intact?)."""
    import bit_weight_gemv_q4_b200 as q4

    t = torch()
    if ws is None:
        ws = workspace(bits, N, K, max(M, 1))
    full = t.full((M * N + 2 * guard,), float("nan"), dtype=t.float32, device="cuda")
    y = full[guard: guard + M * N]
    fn = q4.q4_gemv if bits == 4 else q4.q8_gemv
    fn(packed, N, K, x_dev, M, y, ws)
    q4.q4_workspace_check(ws)
    t.cuda.synchronize()
    f = full.cpu().numpy()
    guards_ok = bool(np.all(np.isnan(f[:guard])) and np.all(np.isnan(f[guard + M * N:])))
    return f[guard: guard + M * N].reshape(M, N), guards_ok


def assert_parity(y, q, s, x, bits, rel=1e-3, abs_=1e-6):
    """|y - y_ref| <= rel * sum|w x| + abs_ element by element (fp64 oracle)."""
    y_ref, B = oracle.gemv(bits, q, s, x)
    ok, err, bound = oracle.within_tolerance(y, y_ref, B, rel, abs_)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        details = [(tuple(i), float(y[tuple(i)]), float(y_ref[tuple(i)]), float(bound[tuple(i)])) for i in idx]
        raise AssertionError(f"{(~ok).sum()} of {ok.size} outside tolerance; first (idx, y, y_ref, bound): {details}")
    return float((err / np.maximum(B, 1e-30)).max()) if B.size else 0.0


def degenerate_rows(bits, N, K, seed=3):
    """Canonical q/s with degenerate rows: every fourth row all zero (nonzero
    scales), the next holds a single nonzero code, the next is zero except for
    one group, the rest random.  The tolerance allows only 1e-6 on a zero row."""
    q, s = synth.tensor(bits, seed, 40, N, K)
    q = q.copy()
    rng = np.random.default_rng(seed)
    for r in range(N):
        kind = r % 4
        if kind == 3:
            continue
        q[r] = 0
        if kind == 1:
            k = int(rng.integers(0, K))
            v = 7 if bits == 4 else 127
            if bits == 4:
                q[r, k // 2] = (v & 0xF) << (4 * (k % 2))
            else:
                q[r, k] = v
        elif kind == 2:
            g = int(rng.integers(0, K // 32))
            vals = rng.integers(-8, 8, 32) if bits == 4 else rng.integers(-127, 128, 32)
            if bits == 4:
                nib = (vals & 0xF).astype(np.uint8)
                q[r, 16 * g: 16 * g + 16] = nib[0::2] | (nib[1::2] << 4)
            else:
                q[r, 32 * g: 32 * g + 32] = vals.astype(np.int8)
    return q, s

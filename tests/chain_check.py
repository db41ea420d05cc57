"""Element-wise parity of a dependent decode chain run on the GPU, op by op,
each op checked on the GPU's own inputs (shared by the chain tests).

* product: every output (or a sample of rows) within the product tolerance
  |y - y_ref| <= 1e-3 sum|w x| + 1e-6 of the fp64 oracle on the bf16
  activations the GPU fed it;
* residual + RMSNorm: the residual stream is replayed in fp32 from the GPU's
  own product outputs (the GPU adds in fp32 too, so the replay is exact and
  the final stream must equal the GPU's bitwise); the bf16 activations must
  equal the oracle's rounding of h / rms * gamma (fp64) except within a
  relative window of a rounding tie, where the fp32 computation may round
  either way;
* SwiGLU: the bf16 activations must equal the oracle's rounding of
  silu(g) * u on the GPU's own gate|up output, outside the tie window.
"""
from __future__ import annotations

import numpy as np

import oracle
from oracle import chain as OC
from bit_weight_gemv_q4_b200 import synth

NORM_TIE = 2.0 ** -17   # the fp32 mean square and two products
SWIGLU_TIE = 2.0 ** -19  # expf, one division, one product


def _host(t):
    return t.detach().cpu().numpy().copy()


def check(ch, sample_rows: int | None = None, seed_rows: int = 1):
    """ch: a workloads.DeviceChain after run() and check().  sample_rows:
    None checks every output row of every product, else that many rows per
    product (the first and last rows, rows around a tile boundary, the rest
    seeded).  Returns a summary dict; raises AssertionError on a mismatch."""
    import bit_weight_gemv_q4_b200 as q4

    M, seed = ch.M, ch.seed
    cache = {}

    def get(t, dtype, shape):
        key = (t.data_ptr(), dtype)
        if key not in cache:
            a = _host(t)
            cache[key] = a.view(dtype).reshape(shape)
        return cache[key]

    rng = np.random.default_rng(seed_rows)
    h32 = None
    stats = {"products": 0, "rows": 0, "norms": 0, "swiglus": 0, "worst_rel": 0.0, "tie_diffs": 0, "values": 0}
    pi = 0
    for kind, bits, N, K, packed, inp, out, resid in ch.ops:
        if kind == q4.Q4_OP_PRODUCT:
            t = ch.w.tensors[pi]
            pi += 1
            x = get(inp, np.uint16, (M, K))
            y = get(out, np.float32, (M, N))
            if sample_rows is None or sample_rows >= N:
                rows = np.arange(N)
                q, s = synth.tensor(t.bits, seed, t.tensor_id, N, K)
                y_ref, B = oracle.gemv(t.bits, q, s, x)
            else:
                fixed = [0, N - 1, min(31, N - 1), min(32, N - 1)]
                rows = np.unique(np.concatenate([fixed, rng.choice(N, sample_rows - len(fixed), replace=False)]))
                y_ref = np.empty((M, rows.size))
                B = np.empty((M, rows.size))
                for j, r in enumerate(rows):
                    q, s = synth.tensor(t.bits, seed, t.tensor_id, N, K, row0=int(r), nrows=1)
                    yr, br = oracle.gemv(t.bits, q, s, x)
                    y_ref[:, j], B[:, j] = yr[:, 0], br[:, 0]
            got = y[:, rows].astype(np.float64)
            ok, err, bound = oracle.within_tolerance(got, y_ref, B)
            if not ok.all():
                m, j = np.argwhere(~ok)[0]
                raise AssertionError(f"product {t.name}: {(~ok).sum()} outputs outside tolerance, first row "
                                     f"{rows[j]} m {m}: {got[m, j]} vs {y_ref[m, j]} (bound {bound[m, j]})")
            stats["products"] += 1
            stats["rows"] += rows.size
            stats["worst_rel"] = max(stats["worst_rel"], float((err / np.maximum(B, 1e-30)).max()))
        elif kind == q4.Q4_OP_RESIDUAL_RMSNORM:
            yv = get(inp, np.float32, (M, N)) if inp is not None else np.zeros((M, N), np.float32)
            if bits == 1:
                h32 = yv.copy()
            elif inp is not None:
                h32 = (h32 + yv).astype(np.float32)  # fp32 addition, as on the GPU
            gamma = OC.bf16_value(get(packed, np.uint16, (N,))) if packed is not None else None
            _, z = OC.residual_rmsnorm(None, h32.astype(np.float64), gamma)
            x = get(out, np.uint16, (M, N))
            diff = x != OC.bf16_bits(z)
            bad = diff & ~OC.near_bf16_tie(z, NORM_TIE)
            if bad.any():
                m, k = np.argwhere(bad)[0]
                raise AssertionError(f"RMSNorm op {stats['norms']}: {bad.sum()} activations differ outside the tie "
                                     f"window, first m {m} k {k}: {x[m, k]:#06x} vs {OC.bf16_bits(z)[m, k]:#06x}")
            stats["norms"] += 1
            stats["tie_diffs"] += int(diff.sum())
            stats["values"] += diff.size
        else:
            ygu = get(inp, np.float32, (M, 2 * N))
            z = OC.swiglu(ygu.astype(np.float64), N)
            x = get(out, np.uint16, (M, N))
            diff = x != OC.bf16_bits(z)
            bad = diff & ~OC.near_bf16_tie(z, SWIGLU_TIE)
            if bad.any():
                m, k = np.argwhere(bad)[0]
                raise AssertionError(f"SwiGLU op {stats['swiglus']}: {bad.sum()} activations differ outside the tie "
                                     f"window, first m {m} k {k}")
            stats["swiglus"] += 1
            stats["tie_diffs"] += int(diff.sum())
            stats["values"] += diff.size
    if h32 is not None:
        h_gpu = _host(ch.h).reshape(h32.shape)
        assert np.array_equal(h_gpu, h32), "the final residual stream differs from its fp32 replay"
    return stats

"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test targets a mistake the oracle could plausibly make: a wrong nibble
order or sign, a wrong scale index (k/32), a dropped or transposed operand,
accumulation in the wrong precision.
"""
import json
import os

import numpy as np
import pytest

import oracle
from bit_weight_gemv_q4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# helpers that build canonical inputs from explicit integer values
# ----------------------------------------------------------------------------
def pack_canonical_q4(qvals: np.ndarray) -> np.ndarray:
    """[N][K] ints in [-8, 7] -> canonical [N][K/2] bytes (low nibble = even k)."""
    nib = (qvals.astype(np.int64) & 0xF).astype(np.uint8)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def f16_bits(vals) -> np.ndarray:
    return np.asarray(vals, dtype=np.float16).view(np.uint16)


def bf16_bits_exact(vals) -> np.ndarray:
    """bf16 bits of values that are exactly representable in bf16."""
    f = np.asarray(vals, dtype=np.float32)
    b = f.view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not exact in bf16"
    return (b >> 16).astype(np.uint16)


def bf16_to_f64_lib(bits: np.ndarray) -> np.ndarray:
    """bf16 is by definition the upper half of an IEEE binary32."""
    with np.errstate(invalid="ignore"):
        return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_to_f64_lib(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def decode_q4_numpy(q: np.ndarray, K: int) -> np.ndarray:
    lo = (q & 0xF).astype(np.int64)
    hi = (q >> 4).astype(np.int64)
    out = np.empty((q.shape[0], K), dtype=np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return np.where(out >= 8, out - 16, out)


# ----------------------------------------------------------------------------
# element decoders
# ----------------------------------------------------------------------------
def test_f16_decoder_all_patterns_match_numpy():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = f16_to_f64_lib(bits)
    got = np.array([oracle.f16_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zero is kept
    assert np.signbit(oracle.f16_value(0x8000))


def test_bf16_decoder_all_patterns_match_binary32_upper_half():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bf16_to_f64_lib(bits)
    got = oracle.bf16_array(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_q4_nibble_table_golden():
    table = {}
    with open(os.path.join(GOLDEN, "q4_nibble_table.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            table[int(a)] = int(b)
    assert sorted(table) == list(range(16))
    # every byte, both positions
    for byte in range(256):
        row = np.array([byte], dtype=np.uint8)
        assert oracle.q4_value(row, 0) == table[byte & 0xF]
        assert oracle.q4_value(row, 1) == table[byte >> 4]


# ----------------------------------------------------------------------------
# hand-worked products
# ----------------------------------------------------------------------------
def _hand_inputs(ex):
    N, K, M, bits = ex["N"], ex["K"], ex["M"], ex["bits"]
    q = np.zeros((N, K), dtype=np.int64)
    if ex["name"] == "q4_two_rows_two_groups":
        q[0, :32] = 1
        q[0, 32] = -8
        q[0, 63] = 7
        q[1, :32] = -1
        q[1, 32::2] = 2
        q[1, 33::2] = -3
        xb = np.empty((M, K), dtype=np.uint16)
        xb[0, :] = ex["x_bits"]["row0_all"]
        xb[1, :32] = ex["x_bits"]["row1_lo"]
        xb[1, 32:] = ex["x_bits"]["row1_hi"]
    else:
        q[0, :] = np.arange(K) - 16
        q[1, 0] = 127
        q[1, 1] = -127
        xb = np.full((M, K), ex["x_bits"]["rest"], dtype=np.uint16)
        xb[0, 0] = ex["x_bits"]["k0"]
        xb[0, 1] = ex["x_bits"]["k1"]
    s = np.array(ex["scale_bits"], dtype=np.uint16)
    # the bit patterns in the fixture are the values printed beside them
    assert np.array_equal(f16_to_f64_lib(s), np.array(ex["scale_values"]))
    qc = pack_canonical_q4(q) if bits == 4 else q.astype(np.int8)
    return qc, s, xb


@pytest.mark.parametrize("idx", [0, 1])
def test_hand_worked_examples(idx):
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        ex = json.load(f)["examples"][idx]
    qc, s, xb = _hand_inputs(ex)
    y, B = oracle.gemv(ex["bits"], qc, s, xb)
    assert np.array_equal(y, np.array(ex["y"]))
    assert np.array_equal(B, np.array(ex["B"]))


# ----------------------------------------------------------------------------
# closed forms and invariants on random inputs
# ----------------------------------------------------------------------------
def _rand_inputs(bits, N, K, M, seed=7, tid=3):
    q, s = synth.tensor(bits, seed, tid, N, K)
    x = synth.activations(seed, synth.act_stream(tid), M, K)
    return q, s, x


@pytest.mark.parametrize("bits", [4, 8])
def test_one_hot_activation_selects_one_weight(bits):
    N, K = 13, 96
    q, s, _ = _rand_inputs(bits, N, K, 1)
    qi = decode_q4_numpy(q, K) if bits == 4 else q.astype(np.int64)
    sv = f16_to_f64_lib(s)
    one = bf16_bits_exact([1.0])[0]
    for k in [0, 1, 31, 32, 33, 63, 64, 95]:
        x = np.zeros((1, K), dtype=np.uint16)
        x[0, k] = one
        y, B = oracle.gemv(bits, q, s, x)
        expect = sv[:, k // 32] * qi[:, k]
        assert np.array_equal(y[0], expect), k
        assert np.array_equal(B[0], np.abs(expect)), k


@pytest.mark.parametrize("bits", [4, 8])
def test_zero_scales_give_zero(bits):
    q, s, x = _rand_inputs(bits, 9, 64, 3)
    y, B = oracle.gemv(bits, q, np.zeros_like(s), x)
    assert np.all(y == 0) and np.all(B == 0)


@pytest.mark.parametrize("c", [-8, -3, 1, 7])
def test_constant_weights_closed_form(c):
    """q = c everywhere: y[m][n] = c * sum_g s[n][g] * (sum of x over group g)."""
    N, K, M = 5, 160, 2
    _, s, x = _rand_inputs(4, N, K, M)
    q = pack_canonical_q4(np.full((N, K), c))
    y, B = oracle.gemv(4, q, s, x)
    xv = bf16_to_f64_lib(x)
    gsum = xv.reshape(M, K // 32, 32).sum(axis=2)  # [M][G]
    expect = c * (gsum @ f16_to_f64_lib(s).T)  # [M][N]
    assert np.allclose(y, expect, rtol=0, atol=1e-12 * (B.max() + 1))


@pytest.mark.parametrize("bits", [4, 8])
def test_linearity_in_x(bits):
    N, K, M = 11, 128, 2
    q, s, x = _rand_inputs(bits, N, K, M)
    y, B = oracle.gemv(bits, q, s, x)
    # doubling a bf16 is exact (exponent + 1), and so is doubling the fp64 sum
    x2 = bf16_bits_exact(2.0 * bf16_to_f64_lib(x).astype(np.float32))
    y2, B2 = oracle.gemv(bits, q, s, x2)
    assert np.array_equal(y2, 2 * y) and np.array_equal(B2, 2 * B)
    # additivity on disjoint supports (so x1 + x2 is exact)
    x1 = x.copy()
    x1[:, 1::2] = 0
    xo = x.copy()
    xo[:, 0::2] = 0
    ya, _ = oracle.gemv(bits, q, s, x1)
    yb, _ = oracle.gemv(bits, q, s, xo)
    assert np.allclose(ya + yb, y, rtol=0, atol=1e-12 * (B.max() + 1))
    # |y| <= B (triangle inequality), B >= 0
    assert np.all(np.abs(y) <= B) and np.all(B >= 0)


@pytest.mark.parametrize("bits,N,K,M", [(4, 7, 32, 1), (4, 16, 256, 4), (8, 9, 96, 3), (8, 33, 64, 2)])
def test_matches_library_matmul_on_dense_dequantisation(bits, N, K, M):
    """Special case that reduces to a library routine: decode the integers with
    numpy, scale by the numpy fp16 value, and multiply with numpy's matmul."""
    q, s, x = _rand_inputs(bits, N, K, M, seed=11)
    qi = decode_q4_numpy(q, K) if bits == 4 else q.astype(np.int64)
    W = qi * np.repeat(f16_to_f64_lib(s), 32, axis=1)
    X = bf16_to_f64_lib(x)
    y_lib = X @ W.T
    b_lib = np.abs(X) @ np.abs(W).T
    y, B = oracle.gemv(bits, q, s, x)
    tol = 4 * K * 2.0**-53 * b_lib + 1e-300
    assert np.all(np.abs(y - y_lib) <= tol)
    assert np.all(np.abs(B - b_lib) <= tol)
    # the oracle's dense dequantisation is the same matrix
    assert np.array_equal(oracle.dequantize(bits, q, s), W)


def test_rows_are_transposed_correctly():
    """Non-square shape with distinct rows: swapping N and K or reading x by
    column would change the shape or the values."""
    N, K, M = 3, 64, 2
    qvals = np.zeros((N, K), dtype=np.int64)
    qvals[0, 5] = 3
    qvals[1, 40] = -2
    qvals[2, 63] = 7
    s = f16_bits(np.ones((N, K // 32)))
    x = np.zeros((M, K), dtype=np.uint16)
    x[0, 5] = bf16_bits_exact([2.0])[0]
    x[1, 40] = bf16_bits_exact([0.5])[0]
    x[1, 63] = bf16_bits_exact([-1.0])[0]
    y, _ = oracle.gemv(4, pack_canonical_q4(qvals), s, x)
    assert y.shape == (M, N)
    assert np.array_equal(y, np.array([[6.0, 0.0, 0.0], [0.0, -1.0, -7.0]]))


def test_accumulation_is_fp64_not_fp32():
    """1 + many tiny terms: an fp32 accumulator would lose the tiny terms."""
    N, K = 1, 4096
    qvals = np.ones((N, K), dtype=np.int64)
    s = f16_bits(np.ones((N, K // 32)))
    x = np.full((1, K), bf16_bits_exact([2.0**-30])[0], dtype=np.uint16)
    x[0, 0] = bf16_bits_exact([1.0])[0]
    y, _ = oracle.gemv(4, pack_canonical_q4(qvals), s, x)
    assert y[0, 0] == 1.0 + (K - 1) * 2.0**-30


def test_scale_subnormals_and_negative_scales():
    N, K = 2, 64
    qvals = np.full((N, K), 7, dtype=np.int64)
    s = np.array([[0x0001, 0x03FF], [0x8400, 0x0000]], dtype=np.uint16)  # min subnormal, max subnormal, -min normal, 0
    x = np.full((1, K), bf16_bits_exact([1.0])[0], dtype=np.uint16)
    y, _ = oracle.gemv(4, pack_canonical_q4(qvals), s, x)
    sv = f16_to_f64_lib(s)
    assert np.array_equal(y[0], 7 * 32 * sv.sum(axis=1))


def test_empty_sum_is_zero():
    """K = 0: every output is the empty sum."""
    q = np.zeros((3, 0), dtype=np.uint8)
    s = np.zeros((3, 0), dtype=np.uint16)
    x = np.zeros((2, 0), dtype=np.uint16)
    y, B = oracle.gemv(4, q, s, x)
    assert y.shape == (2, 3) and np.all(y == 0) and np.all(B == 0)

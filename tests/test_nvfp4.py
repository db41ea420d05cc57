"""NVFP4 weights: the oracle's decode pinned by the format's published value
sets and closed forms (CPU); the packer's round trip (CPU); device decode and
products against the oracle (GPU)."""
import numpy as np
import pytest

from oracle import nvfp4 as ON
from bit_weight_gemv_q4_b200 import synth

RNG = np.random.default_rng(44)


# ---------------------------------------------------------------- oracle pins
def test_e2m1_value_set():
    # the sixteen E2M1 numbers, codes 0..15: 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives
    assert ON.E2M1.tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    assert np.signbit(ON.E2M1[8])


def test_e4m3_landmarks():
    assert ON.e4m3_value(0x38) == 1.0
    assert ON.e4m3_value(0x7E) == 448.0          # largest finite
    assert ON.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal
    assert ON.e4m3_value(0x08) == 2.0 ** -6      # smallest normal
    assert ON.e4m3_value(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert np.isnan(ON.e4m3_value(0x7F)) and np.isnan(ON.e4m3_value(0xFF))
    pos = ON.E4M3[:0x7F]
    assert np.all(np.diff(pos) > 0)  # the finite positive codes are increasing
    assert np.array_equal(ON.E4M3[0x80:0xFF], -pos)


def test_one_hot_weights_and_products():
    N, K = 4, 64
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.full((N, K // 16), 0x38, dtype=np.uint8)  # 1.0
    codes[2, 5] = 0x70  # row 2, k = 11: code 7 (= 6.0) in the high nibble
    scales[2, 0] = 0x40  # block 0 of row 2: 2.0
    w = ON.dequantize(codes, scales, 0.5, K)
    assert w[2, 11] == 0.5 * 2.0 * 6.0 and np.count_nonzero(w) == 1
    x = np.zeros((1, K), dtype=np.uint16)
    x[0, 11] = 0x4040  # 3.0
    y, B = ON.gemv(codes, scales, 0.5, x)
    assert y[0].tolist() == [0.0, 0.0, 18.0, 0.0] and B[0, 2] == 18.0


def test_product_brute_force():
    N, K, M = 5, 96, 3
    codes = RNG.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = RNG.integers(0x20, 0x50, (N, K // 16), dtype=np.uint8)
    xf = RNG.normal(0, 1, (M, K))
    x = synth.f64_to_bf16_bits(xf.ravel()).reshape(M, K)
    xv = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y, B = ON.gemv(codes, scales, 0.125, x)
    for m in range(M):
        for n in range(N):
            acc = absacc = 0.0
            for k in range(K):
                nib = (codes[n, k // 2] >> (4 * (k % 2))) & 0xF
                w = 0.125 * ON.e4m3_value(int(scales[n, k // 16])) * ON.e2m1_value(int(nib))
                acc += w * xv[m, k]
                absacc += abs(w * xv[m, k])
            assert np.isclose(y[m, n], acc, rtol=1e-13, atol=1e-15)
            assert np.isclose(B[m, n], absacc, rtol=1e-13, atol=1e-15)


def test_generator_ranges():
    c, s, t = synth.nvfp4_tensor(0, 7, 33, 128)
    assert c.shape == (33, 64) and s.shape == (33, 8)
    assert s.min() >= 0x28 and s.max() <= 0x47 and t == synth.NVFP4_TENSOR_SCALE
    vals = ON.E4M3[s]
    assert np.all(np.isfinite(vals)) and vals.min() == 0.25 or vals.min() > 0.25

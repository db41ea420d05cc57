"""The offline quantiser: the oracle pinned against exact rational arithmetic
and hand-worked groups (CPU), the library's host quantiser bit-exact against
the oracle (CPU), and the device quantiser bit-exact against it (GPU)."""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import quantize as OQ
import oracle

RNG = np.random.default_rng(2024)


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    from bit_weight_gemv_q4_b200 import synth

    return synth.f64_to_bf16_bits(np.asarray(a, dtype=np.float64).ravel()).reshape(np.shape(a))


def _exact_round(fr: Fraction, mant_bits: int, emin: int) -> Fraction:
    """Nearest binary float with mant_bits significand bits and minimum
    exponent emin (subnormals below), ties to even; exact arithmetic."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - (mant_bits - 1))
    t = a / ulp
    n = t.numerator // t.denominator
    rem = t - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def _f16_of_f32(v: Fraction) -> Fraction:
    r = _exact_round(v, 11, -14)
    return max(min(r, Fraction(65504)), Fraction(-65504))


def _f16_bits_value(b: int) -> Fraction:
    return Fraction(float(np.array([b], dtype=np.uint16).view(np.float16)[0]))


def _groups(N=6, K=128, scale=0.02):
    w = RNG.normal(0, scale, (N, K))
    w[0, :32] = 0.0                      # an all-zero group
    w[1, 32:64] *= 1e-30                 # a group whose scale rounds to zero or a subnormal
    w[2, 64:96] = np.round(w[2, 64:96] / 0.01) * 0.01  # many near-ties
    w[3, :32] = RNG.choice([-3.0, 3.0], 32)            # equal magnitudes, both signs
    return _bf16_bits(w)


# ---------------------------------------------------------------- oracle pins
@pytest.mark.parametrize("bits,mode", [(4, OQ.ABSMAX), (4, OQ.SIGNED_MAX), (8, OQ.ABSMAX)])
def test_scales_follow_the_stated_rounding_exactly(bits, mode):
    wb = _groups()
    q, s = OQ.quantize_ints(bits, mode, wb)
    wf = OQ.bf16_to_f32(wb).astype(np.float64)
    N, K = wb.shape
    for n in range(N):
        for g in range(K // 32):
            grp = [Fraction(float(v)) for v in wf[n, 32 * g: 32 * g + 32]]
            if mode == OQ.ABSMAX:
                amax = max(abs(v) for v in grp)
                s32 = _exact_round(amax / (7 if bits == 4 else 127), 24, -126)
            else:
                wm = max(grp, key=abs)  # first of the largest magnitude
                s32 = _exact_round(wm / -8, 24, -126)
            assert _f16_bits_value(int(s[n, g])) == _f16_of_f32(s32), (n, g)


@pytest.mark.parametrize("bits,mode", [(4, OQ.ABSMAX), (4, OQ.SIGNED_MAX), (8, OQ.ABSMAX)])
def test_codes_are_the_nearest_in_range(bits, mode):
    """Brute force in exact arithmetic: each code is the integer in range
    nearest to the exact quotient w / s, ties to even."""
    wb = _groups()
    q, s = OQ.quantize_ints(bits, mode, wb)
    lo, hi = OQ.code_range(bits, mode)
    wf = OQ.bf16_to_f32(wb).astype(np.float64)
    N, K = wb.shape
    for n in range(N):
        for k in range(K):
            sv = _f16_bits_value(int(s[n, k // 32]))
            if sv == 0:
                assert q[n, k] == 0
                continue
            r = Fraction(float(wf[n, k])) / sv
            best = min(range(lo, hi + 1), key=lambda j: (abs(r - j), j % 2))
            assert q[n, k] == best, (n, k, float(r), q[n, k], best)


def test_hand_worked_group():
    """w = (1, -1/2, 1/4, 1/8, 0, 1/16, 0...): absmax q4 scale fp16(1/7) =
    585/4096 (0x3092), quotients 7.0017, -3.5009, 1.7504, 0.8752, 0, 0.4376
    -> codes 7, -4, 2, 1, 0, 0; signed q4 scale -1/8 (0xB000) -> codes
    -8, 4, -2, -1, 0, and rint(-0.5) = 0."""
    w = np.zeros((1, 32))
    w[0, :6] = [1.0, -0.5, 0.25, 0.125, 0.0, 0.0625]
    wb = _bf16_bits(w)
    q, s = OQ.quantize_ints(4, OQ.ABSMAX, wb)
    assert int(s[0, 0]) == 0x3092
    assert q[0, :6].tolist() == [7, -4, 2, 1, 0, 0] and not q[0, 6:].any()
    q, s = OQ.quantize_ints(4, OQ.SIGNED_MAX, wb)
    assert int(s[0, 0]) == 0xB000
    assert q[0, :6].tolist() == [-8, 4, -2, -1, 0, 0]


def test_extreme_value_gets_the_extreme_code():
    wb = _groups(N=8, K=256)
    wf = OQ.bf16_to_f32(wb).reshape(8, 8, 32)
    q, s = OQ.quantize_ints(4, OQ.ABSMAX, wb)
    q = q.reshape(8, 8, 32)
    q8, _ = OQ.quantize_ints(8, OQ.ABSMAX, wb)
    q8 = q8.reshape(8, 8, 32)
    qs, ss = OQ.quantize_ints(4, OQ.SIGNED_MAX, wb)
    qs = qs.reshape(8, 8, 32)
    for n in range(8):
        for g in range(8):
            if not wf[n, g].any() or s[n, g] == 0:
                continue
            i = int(np.abs(wf[n, g]).argmax())
            assert abs(q[n, g, i]) == 7 and abs(q8[n, g, i]) == 127
            if ss[n, g]:
                assert qs[n, g, i] == -8


def test_reconstruction_error_bounds():
    """Absmax: at most half a step, plus the fp16 rounding of the scale (2^-11
    relative) carried to the largest code.  Signed: values of the other sign
    than the extreme one reach up to 8 steps and are clamped to code 7, so up
    to one step; the rest at most half a step."""
    wb = _bf16_bits(RNG.normal(0, 0.02, (16, 512)))
    wf = OQ.bf16_to_f32(wb).astype(np.float64)
    for bits, mode in [(4, OQ.ABSMAX), (4, OQ.SIGNED_MAX), (8, OQ.ABSMAX)]:
        q, s = OQ.quantize_ints(bits, mode, wb)
        sf = s.view(np.float16).astype(np.float64).repeat(32, axis=1)
        err = np.abs(wf - sf * q) / np.abs(sf)
        if mode == OQ.ABSMAX:
            qmax = 7 if bits == 4 else 127
            assert err.max() <= 0.5 + qmax * 2.0 ** -11
        else:
            assert err.max() <= 1.0 + 8 * 2.0 ** -11
            assert err[q != 7].max() <= 0.5 + 8 * 2.0 ** -11


def test_zero_and_degenerate_groups():
    w = np.zeros((2, 64))
    w[1, 32:] = 1e-38  # scale below every fp16 subnormal: rounds to 0
    q, s = OQ.quantize_ints(4, OQ.ABSMAX, _bf16_bits(w))
    assert not q.any() and not s.any()


def test_canonical_layout_matches_the_nibble_convention():
    wb = _bf16_bits(RNG.normal(0, 1.0, (3, 64)))
    q, s = OQ.quantize_ints(4, OQ.SIGNED_MAX, wb)
    c = OQ.to_canonical(4, q)
    for n in range(3):
        for k in range(64):
            assert oracle.q4_value(c[n], k) == q[n, k]
    c8 = OQ.to_canonical(8, np.clip(q * 18, -127, 127))
    assert c8.dtype == np.int8 and np.array_equal(c8.astype(np.int32), np.clip(q * 18, -127, 127))


# ---------------------------------------------------------------- library vs oracle
def _finite_bf16_patterns(N, K, seed):
    """Every kind of finite bf16: random bit patterns (subnormals, huge values,
    signed zeros) with the inf/NaN exponent replaced."""
    rng = np.random.default_rng(seed)
    b = rng.integers(0, 1 << 16, (N, K), dtype=np.uint32).astype(np.uint16)
    bad = (b & 0x7F80) == 0x7F80
    b[bad] &= 0xBFFF  # exponent 0x7F -> 0x3F
    b[0, :32] = 0x8000  # a group of negative zeros
    b[0, 32:64] = 0x0001  # smallest subnormals
    return b


def _weight_cases():
    yield "normal", _bf16_bits(RNG.normal(0, 0.02, (37, 256)))
    yield "patterns", _finite_bf16_patterns(23, 128, 7)
    yield "ties", _bf16_bits(np.round(RNG.normal(0, 1, (9, 64)) * 4) / 8)


@pytest.mark.parametrize("bits,mode", [(4, OQ.ABSMAX), (4, OQ.SIGNED_MAX), (8, OQ.ABSMAX)])
def test_host_quantiser_is_bit_exact(bits, mode):
    import bit_weight_gemv_q4_b200 as q4

    for name, wb in _weight_cases():
        q, s = q4.q4_quantize(bits, mode, wb)
        qo, so = OQ.quantize(bits, mode, wb)
        assert np.array_equal(s, so), name
        assert np.array_equal(q.view(np.uint8), qo.view(np.uint8)), name


def test_quantiser_argument_errors():
    import bit_weight_gemv_q4_b200 as q4

    w = np.zeros((2, 64), dtype=np.uint16)
    with pytest.raises(q4.Q4Error):
        q4.q4_quantize(8, q4.Q4_QUANT_SIGNED_MAX, w)  # signed mode is q4 only
    with pytest.raises(q4.Q4Error):
        q4.q4_quantize(5, q4.Q4_QUANT_ABSMAX, w)
    with pytest.raises(q4.Q4Error):
        q4.q4_quantize(4, q4.Q4_QUANT_ABSMAX, np.zeros((2, 48), dtype=np.uint16))  # K % 32
    q, s = q4.q4_quantize(4, q4.Q4_QUANT_ABSMAX, np.zeros((0, 64), dtype=np.uint16))
    assert q.size == 0 and s.size == 0


@pytest.mark.gpu
@pytest.mark.parametrize("bits,mode", [(4, OQ.ABSMAX), (4, OQ.SIGNED_MAX), (8, OQ.ABSMAX)])
def test_device_quantiser_is_bit_exact(cuda_device, bits, mode):
    import torch

    import bit_weight_gemv_q4_b200 as q4

    for name, wb in _weight_cases():
        N, K = wb.shape
        w = torch.from_numpy(wb.view(np.int16)).cuda()
        q = torch.zeros(N * (K // 2 if bits == 4 else K), dtype=torch.uint8, device="cuda")
        s = torch.zeros(N * (K // 32), dtype=torch.int16, device="cuda")
        q4.q4_quantize_device(bits, mode, w, N, K, q, s)
        torch.cuda.synchronize()
        qo, so = OQ.quantize(bits, mode, wb)
        assert np.array_equal(s.cpu().numpy().view(np.uint16).reshape(N, K // 32), so), name
        assert np.array_equal(q.cpu().numpy().reshape(qo.shape), qo.view(np.uint8)), name


@pytest.mark.gpu
@pytest.mark.parametrize("bits,mode", [(4, OQ.SIGNED_MAX), (8, OQ.ABSMAX)])
def test_quantise_pack_and_multiply_on_the_device(cuda_device, bits, mode):
    """bf16 weights -> device quantiser -> device packer -> product, against
    the oracle product of the oracle's quantisation of the same weights."""
    import torch

    import bit_weight_gemv_q4_b200 as q4
    from bit_weight_gemv_q4_b200 import synth

    N, K, M = 300, 1024, 2
    wb = _bf16_bits(RNG.normal(0, 0.02, (N, K)))
    w = torch.from_numpy(wb.view(np.int16)).cuda()
    q = torch.zeros(N * (K // 2 if bits == 4 else K), dtype=torch.uint8, device="cuda")
    s = torch.zeros(N * (K // 32), dtype=torch.int16, device="cuda")
    q4.q4_quantize_device(bits, mode, w, N, K, q, s)
    packed = torch.zeros(q4.q4_packed_bytes(bits, N, K), dtype=torch.uint8, device="cuda")
    q4.q4_pack_weights_device(bits, q, s, N, K, packed)
    x = synth.activations(9, synth.act_stream(77), M, K)
    xd = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda()
    y = torch.empty(M * N, dtype=torch.float32, device="cuda")
    ws = torch.zeros(q4.q4_gemv_workspace_bytes(bits, N, K, M), dtype=torch.uint8, device="cuda")
    (q4.q4_gemv if bits == 4 else q4.q8_gemv)(packed, N, K, xd, M, y, ws)
    q4.q4_workspace_check(ws)
    qo, so = OQ.quantize(bits, mode, wb)
    y_ref, B = oracle.gemv(bits, qo, so, x)
    ok, _, _ = oracle.within_tolerance(y.cpu().numpy().reshape(M, N).astype(np.float64), y_ref, B)
    assert ok.all()

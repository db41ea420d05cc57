"""NVFP4 weights: the oracle's decode pinned by the format's published value
sets and closed forms (CPU); the packer's round trip (CPU); device decode and
products against the oracle (GPU)."""
import numpy as np
import pytest

from oracle import nvfp4 as ON
from bit_weight_gemv_q4_b200 import synth, workloads

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


# ---------------------------------------------------------------- packer (CPU)
def _expected_packed(codes, scales, t, N, K):
    """The packed bytes by the documented placement, written as the map from
    each (row, column) to its byte: tile t = row // 32, half h, slot (gi, ti),
    word j = 2G + e, register r = 2 * (column bit 1) + (row bit 3)."""
    T, C = -(-N // 32), K // 64
    out = np.zeros(T * C * 1152 + 16, dtype=np.uint8)
    rows = np.arange(N)[:, None]
    cols = np.arange(0, K, 2)[None, :]  # even columns: one canonical byte each
    tt, rr = rows // 32, rows % 32
    h, gi, up = rr // 16, rr % 8, (rr % 16) // 8
    c, cc = cols // 64, cols % 64
    G, ti, e, rhi = cc // 32, (cc % 32) // 8, (cc % 8) // 4, (cc % 4) // 2
    off = (tt * C + c) * 1152 + 512 * h + 16 * (4 * gi + ti) + 4 * (2 * G + e) + (2 * rhi + up)
    out[off.ravel()] = codes.ravel()
    blk = np.arange(K // 16)[None, :]
    c, bb = blk // 4, blk % 4
    off = (tt * C + c) * 1152 + 1024 + 8 * (2 * gi + bb % 2) + 4 * h + 2 * (bb // 2) + up
    out[off.ravel()] = scales.ravel()
    out[T * C * 1152: T * C * 1152 + 4] = np.frombuffer(np.float32(t).tobytes(), dtype=np.uint8)
    return out


@pytest.fixture(scope="module")
def q4():
    import bit_weight_gemv_q4_b200 as lib

    return lib


@pytest.mark.parametrize("N,K", [(1, 64), (32, 128), (70, 192), (33, 5120)])
def test_pack_places_every_byte_as_documented(q4, N, K):
    codes = RNG.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = RNG.integers(0, 256, (N, K // 16), dtype=np.uint8)
    packed = q4.q4_pack_nvfp4(codes, scales, 0.375, N, K)
    assert packed.size == q4.q4_nvfp4_packed_bytes(N, K) == -(-N // 32) * (K // 64) * 1152 + 16
    assert np.array_equal(packed, _expected_packed(codes, scales, 0.375, N, K))
    c2, s2, t2 = q4.q4_unpack_nvfp4(packed, N, K)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales) and t2 == 0.375


def test_pack_register_bytes_match_q4_nibble_columns(q4):
    """The columns of NVFP4 register r in word j are those of the q4 format's
    nibbles i = r and r + 4 of the same word: one set of activation fragments
    serves both.  Checked by packing one-hot tensors in both formats."""
    N, K = 32, 64
    for row, col in [(0, 0), (9, 1), (17, 6), (31, 63), (4, 37), (12, 42)]:
        codes = np.zeros((N, K // 2), dtype=np.uint8)
        codes[row, col // 2] = 0x3 << (4 * (col % 2))
        nv = q4.q4_pack_nvfp4(codes, np.zeros((N, K // 16), np.uint8), 1.0, N, K)[:1024]
        q = np.full((N, K // 2), 0, dtype=np.uint8)
        q[row, col // 2] = 0x3 << (4 * (col % 2))
        p4 = q4.q4_pack_weights(4, q, np.zeros((N, K // 32), np.uint16), N, K)[:1024]
        # q4 stores u = q + 8: the one nonzero code is the nibble that differs from 8
        w4 = p4.view(np.uint32)
        nib = (w4[:, None] >> (4 * np.arange(8))[None, :]) & 0xF
        word4, i4 = np.argwhere(nib != 8)[0]
        byte_nv = int(np.flatnonzero(nv)[0])
        word_nv, r = byte_nv // 4, byte_nv % 4
        assert word_nv == word4 and i4 % 4 == r, (row, col)
        # and the same half of the fp16 pair: low nibble <-> nibble i < 4
        assert (nv[byte_nv] & 0xF != 0) == (i4 < 4)


def test_pack_errors(q4):
    with pytest.raises(q4.Q4Error, match="SHAPE"):
        q4.q4_pack_nvfp4(np.zeros((4, 48), np.uint8), np.zeros((4, 6), np.uint8), 1.0, 4, 96)
    assert q4.q4_nvfp4_packed_bytes(4, 96) == 0 and q4.q4_nvfp4_packed_bytes(0, 64) == 16


def test_nvfp4_stream_has_q4_bytes():
    ts = workloads.decode_stream(fused=True)
    assert workloads.total_bytes(workloads.as_nvfp4(ts)) == workloads.total_bytes(ts)


# ---------------------------------------------------------------- device (GPU)
def _gpu():
    import torch

    return torch


def _assert_parity(y, codes, scales, t, x, rel=1e-3, abs_=1e-6):
    import oracle

    y_ref, B = ON.gemv(codes, scales, t, x)
    ok, err, bound = oracle.within_tolerance(y, y_ref, B, rel, abs_)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        details = [(tuple(i), float(y[tuple(i)]), float(y_ref[tuple(i)]), float(bound[tuple(i)])) for i in idx]
        raise AssertionError(f"{(~ok).sum()} of {ok.size} outside tolerance; first (idx, y, y_ref, bound): {details}")


def _dev_bytes(a):
    torch = _gpu()
    a = np.ascontiguousarray(a).view(np.uint8).ravel()
    buf = torch.empty(max(a.size, 16), dtype=torch.uint8, device="cuda")
    if a.size:
        buf[: a.size].copy_(torch.from_numpy(a))
    return buf


def _dev_x(x):
    torch = _gpu()
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("N,K", [(70, 192), (4099, 5120), (1, 64)])
def test_device_pack_equals_host_pack(q4, cuda_device, N, K):
    torch = _gpu()
    codes, scales, t = synth.nvfp4_tensor(3, 61, N, K)
    host = q4.q4_pack_nvfp4(codes, scales, t, N, K)
    out = torch.full((host.size,), 0xAB, dtype=torch.uint8, device="cuda")
    q4.q4_pack_nvfp4_device(_dev_bytes(codes), _dev_bytes(scales), t, N, K, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), host)


@pytest.mark.gpu
def test_device_decode_of_every_code_and_scale(q4, cuda_device):
    """Every E2M1 code against every finite E4M3 scale through the in-register
    conversion: w = t * e4m3 * e2m1, equal to the oracle's fp64 value rounded
    once to fp32 (the fp16 product is exact)."""
    torch = _gpu()
    finite = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], dtype=np.uint8)
    N, K = 254, 512  # every code byte in every row, every finite scale byte in many places
    scales = np.empty((N, K // 16), dtype=np.uint8)
    for r in range(N):
        scales[r] = np.roll(finite, r)[: K // 16]
    codes = np.tile(np.arange(256, dtype=np.uint8), (N, 1))[:, : K // 2]
    t = np.float32(0.8125)
    packed = _dev_bytes(q4.q4_pack_nvfp4(codes, scales, t, N, K))
    w = torch.empty(N * K, dtype=torch.float32, device="cuda")
    q4.q4_nvfp4_dequant_device(packed, N, K, w)
    torch.cuda.synchronize()
    ref = ON.dequantize(codes, scales, t, K).astype(np.float32)
    got = w.cpu().numpy().reshape(N, K)
    assert np.array_equal(got.view(np.uint32) & 0x7FFFFFFF, ref.view(np.uint32) & 0x7FFFFFFF)
    nz = ref != 0
    assert np.array_equal(np.signbit(got[nz]), np.signbit(ref[nz]))


def _stack(q4, specs, M, x_by_k, flags=None):
    """specs: (fmt, N, K, tensor_id); returns (stack, [(fmt, N, K, host data, y)])."""
    torch = _gpu()
    entries, out = [], []
    for fmt, N, K, tid in specs:
        if fmt == workloads.NVFP4:
            c, s, t = synth.nvfp4_tensor(4, tid, N, K)
            packed = _dev_bytes(q4.q4_pack_nvfp4(c, s, t, N, K))
            host = (c, s, t)
        else:
            q, s = synth.tensor(fmt, 4, tid, N, K)
            packed = _dev_bytes(q4.q4_pack_weights(fmt, q, s, N, K))
            host = (q, s)
        y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
        entries.append((fmt, N, K, packed, x_by_k[K][1], y))
        out.append((fmt, N, K, host, y))
    st = q4.layer_stack_create(entries, M, q4.Q4_STACK_INDEPENDENT if flags is None else flags)
    return st, out


def _check_outputs(out, x_by_k, M):
    import gpu_helpers as H

    for fmt, N, K, host, y in out:
        yy = y.cpu().numpy().reshape(M, N)
        assert np.all(np.isfinite(yy))
        if fmt == workloads.NVFP4:
            _assert_parity(yy, *host, x_by_k[K][0])
        else:
            H.assert_parity(yy, host[0], host[1], x_by_k[K][0], fmt)


NV = workloads.NVFP4
STACKS = {
    # stages of four chunks
    "nvfp4": [(NV, 1000, 5120, 71), (NV, 17, 17408, 72), (NV, 4099, 5120, 73), (NV, 64, 256, 74)],
    # q4, q8 and NVFP4 products interleaved, sharing activations (stages of four)
    "mixed": [(4, 1000, 5120, 75), (NV, 3, 5120, 76), (8, 37, 5120, 77), (NV, 7168, 5120, 78), (4, 64, 256, 79),
              (NV, 33, 256, 80)],
    # a K of 128 (two chunks per tile): stages of two
    "su2": [(NV, 100, 128, 81), (4, 40, 128, 82), (NV, 2050, 5120, 83)],
}


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("which", sorted(STACKS))
def test_stream_stack_parity(q4, cuda_device, which, M):
    torch = _gpu()
    specs = STACKS[which]
    x_by_k = {}
    for K in sorted({k for _, _, k, _ in specs}):
        x = synth.activations(4, synth.act_stream(K), M, K)
        x_by_k[K] = (x, _dev_x(x))
    st, out = _stack(q4, specs, M, x_by_k)
    assert st.launches() == 2
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    first = [y.cpu().numpy().copy() for *_, y in out]
    _check_outputs(out, x_by_k, M)
    for *_, y in out:
        y.fill_(float("nan"))
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    for f, (*_, y) in zip(first, out):
        assert np.array_equal(y.cpu().numpy(), f)  # bitwise reproducible
    st.close()


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["wide_range", "huge", "tiny", "zeros", "subnormal"])
@pytest.mark.parametrize("M", [1, 4])
def test_activation_ranges(q4, cuda_device, case, M):
    """The bf16 fallback (no power of two brings x into fp16) and the scaled
    fp16 path, on NVFP4 products."""
    torch = _gpu()
    K = 5120
    x = synth.activations(6, synth.act_stream(44), M, K)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if case == "wide_range":
        xf[:, ::7] *= 2.0 ** 60
        xf[:, 3::11] *= 2.0 ** -60
    elif case == "tiny":
        xf *= 2.0 ** -100
    elif case == "huge":
        xf *= 2.0 ** 100
    elif case == "zeros":
        xf[:] = 0.0
    else:
        xf *= 2.0 ** -128
    x = synth.f64_to_bf16_bits(xf.ravel()).reshape(M, K)
    x_by_k = {K: (x, _dev_x(x))}
    st, out = _stack(q4, [(NV, 160, K, 91), (4, 96, K, 92)], M, x_by_k)
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    if case == "zeros":
        for *_, y in out:
            assert np.all(y.cpu().numpy() == 0.0)
    _check_outputs(out, x_by_k, M)
    st.close()


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 3])
def test_degenerate_rows(q4, cuda_device, M):
    """All-zero code rows, zero block scales, a single nonzero code, negative
    zero codes (0x8): within the tolerance, 1e-6 on a zero row."""
    torch = _gpu()
    N, K = 96, 5120
    codes, scales, t = synth.nvfp4_tensor(5, 93, N, K)
    codes, scales = codes.copy(), scales.copy()
    codes[0::4] = 0
    codes[1::4] = 0x88  # -0, -0
    scales[2::4] = 0
    codes[3::8] = 0
    codes[3::8, 17] = 0x70
    x = synth.activations(5, synth.act_stream(45), M, K)
    y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
    xd = _dev_x(x)
    st = q4.layer_stack_create([(NV, N, K, _dev_bytes(q4.q4_pack_nvfp4(codes, scales, t, N, K)), xd, y)], M,
                               q4.Q4_STACK_INDEPENDENT)
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    yy = y.cpu().numpy().reshape(M, N)
    assert np.all(yy[:, 0::4] == 0) and np.all(yy[:, 1::4] == 0) and np.all(yy[:, 2::4] == 0)
    _assert_parity(yy, codes, scales, t, x)
    st.close()


@pytest.mark.gpu
def test_unsupported_modes_are_refused(q4, cuda_device):
    torch = _gpu()
    N, K = 64, 256
    c, s, t = synth.nvfp4_tensor(1, 94, N, K)
    p = _dev_bytes(q4.q4_pack_nvfp4(c, s, t, N, K))
    x = _dev_x(synth.activations(1, 1, 1, K))
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    for flags in (0, q4.Q4_STACK_GRAPH, q4.Q4_STACK_INDEPENDENT | q4.Q4_STACK_NO_PDL):
        with pytest.raises(q4.Q4Error, match="UNSUPPORTED"):
            q4.layer_stack_create([(NV, N, K, p, x, y)], 1, flags)
    # a q4 product with K % 64 == 32 rules stream mode out
    q, sc = synth.tensor(4, 1, 95, 32, 96)
    p4 = _dev_bytes(q4.q4_pack_weights(4, q, sc, 32, 96))
    x96 = _dev_x(synth.activations(1, 2, 1, 96))
    y96 = torch.empty(32, dtype=torch.float32, device="cuda")
    with pytest.raises(q4.Q4Error, match="UNSUPPORTED"):
        q4.layer_stack_create([(NV, N, K, p, x, y), (4, 32, 96, p4, x96, y96)], 1, q4.Q4_STACK_INDEPENDENT)
    with pytest.raises(q4.Q4Error, match="SHAPE"):
        q4.layer_stack_create([(NV, N, 96, p, x96, y)], 1, q4.Q4_STACK_INDEPENDENT)


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 4])
def test_full_decode_stream_in_nvfp4_sampled(q4, cuda_device, M):
    """The 64-layer decode stream with its 4-bit tensors in NVFP4 (13.7 GB, the
    q4 stream's bytes) in one stream-mode launch; sampled rows of several
    tensors against the oracle."""
    torch = _gpu()
    tensors = workloads.as_nvfp4(workloads.decode_stream(fused=True))
    st = workloads.DeviceStream(tensors, M, flags=q4.Q4_STACK_INDEPENDENT)
    assert st.stack.launches() == 2
    st.run()
    st.check()
    torch.cuda.synchronize()
    rng = np.random.default_rng(M)
    import gpu_helpers as H

    for i in [0, 1, 2, 3, 12, 13, 14, 15, 128, 254, 255, 256]:
        t = tensors[i]
        y = st.y[i].cpu().numpy().reshape(M, t.N)
        assert np.all(np.isfinite(y)), t.name
        x = synth.activations(st.seed, synth.act_stream(workloads.activation_stream_id(t.K)), M, t.K)
        for r in sorted({0, t.N - 1} | set(rng.integers(0, t.N, 6).tolist())):
            if t.bits == NV:
                c, s, ts = synth.nvfp4_tensor(st.seed, t.tensor_id, t.N, t.K, row0=r, nrows=1)
                _assert_parity(y[:, r:r + 1], c, s, ts, x)
            else:
                q, s = synth.tensor(t.bits, st.seed, t.tensor_id, t.N, t.K, row0=r, nrows=1)
                H.assert_parity(y[:, r:r + 1], q, s, x, t.bits)
    st.close()
    torch.cuda.empty_cache()

"""q5 / q6 weights (symmetric, group 32, fp16 scales; the widths between q4
and q8): the packed layout against its written specification and the
packer's round trip (CPU); the device packer, the register decode and the
stream-mode products against the oracle (GPU)."""
import numpy as np
import pytest

import oracle
from oracle import layout
from bit_weight_gemv_q4_b200 import synth, workloads

RNG = np.random.default_rng(56)
RANGE = {5: 16, 6: 32}


@pytest.fixture(scope="module")
def q4():
    import bit_weight_gemv_q4_b200 as lib

    return lib


def _codes(bits, N, K, rng=RNG):
    r = RANGE[bits]
    return rng.integers(-r, r, (N, K)).astype(np.int8)


# ---------------------------------------------------------------- CPU
@pytest.mark.parametrize("bits", [5, 6])
@pytest.mark.parametrize("N,K", [(1, 64), (32, 128), (70, 192), (33, 5120)])
def test_pack_matches_the_layout_specification(q4, bits, N, K):
    q = _codes(bits, N, K)
    s = RNG.integers(0, 1 << 16, (N, K // 32)).astype(np.uint16)
    packed = q4.q4_pack_weights(bits, q, s, N, K)
    cb = {5: 1408, 6: 1664}[bits]
    assert packed.size == q4.q4_packed_bytes(bits, N, K) == -(-N // 32) * (K // 64) * cb
    qd, sd = layout.decode(bits, packed, N, K)
    assert np.array_equal(qd, q.astype(np.int64)) and np.array_equal(sd, s)
    assert layout.padding_is_zero(bits, packed, N, K)
    q2, s2 = q4.q4_unpack_weights(bits, packed, N, K)
    assert np.array_equal(q2, q) and np.array_equal(s2, s)


@pytest.mark.parametrize("bits", [5, 6])
def test_high_bit_positions_fill_the_plane(q4, bits):
    """Every high bit of the plane belongs to exactly one value: the largest
    codes set all of them, the smallest none, and one code sets one field."""
    N, K = 32, 64
    r = RANGE[bits]
    s = np.zeros((N, K // 32), np.uint16)
    hi_lo, hi_hi = 1024, 1024 + (256 if bits == 5 else 512)
    top = q4.q4_pack_weights(bits, np.full((N, K), r - 1, np.int8), s, N, K)
    assert np.all(top[hi_lo:hi_hi] == 0xFF) and np.all(top[:1024] == 0xFF)
    bottom = q4.q4_pack_weights(bits, np.full((N, K), -r, np.int8), s, N, K)
    assert not bottom[hi_lo:hi_hi].any() and not bottom[:1024].any()
    for row, col in [(0, 0), (9, 37), (31, 63), (16, 8)]:
        q = np.full((N, K), -r, np.int8)
        q[row, col] = -r + 16  # u = 16: one high bit (the lowest of the field)
        p = q4.q4_pack_weights(bits, q, s, N, K)
        assert sum(bin(b).count("1") for b in p[hi_lo:hi_hi]) == 1 and not p[:1024].any()


def test_pack_errors(q4):
    with pytest.raises(q4.Q4Error, match="INVALID_ARG"):
        q4.q4_pack_weights(5, np.full((4, 64), 16, np.int8), np.zeros((4, 2), np.uint16), 4, 64)
    with pytest.raises(q4.Q4Error, match="INVALID_ARG"):
        q4.q4_pack_weights(6, np.full((4, 64), -33, np.int8), np.zeros((4, 2), np.uint16), 4, 64)
    with pytest.raises(q4.Q4Error, match="SHAPE"):
        q4.q4_pack_weights(5, np.zeros((4, 96), np.int8), np.zeros((4, 3), np.uint16), 4, 96)
    assert q4.q4_packed_bytes(6, 4, 96) == 0 and q4.q4_packed_bytes(7, 4, 64) == 0


@pytest.mark.parametrize("bits", [5, 6])
def test_oracle_takes_the_plain_definition(bits):
    """q5 / q6 products are s * q * x summed, the q8 definition on narrower
    codes; out-of-range codes are refused."""
    N, K, M = 7, 96, 2
    q = _codes(bits, N, K)
    s = synth.f64_to_f16_bits(RNG.random(N * K // 32) * 0.05).reshape(N, K // 32)
    x = synth.f64_to_bf16_bits(RNG.normal(0, 1, M * K)).reshape(M, K)
    assert np.array_equal(oracle.gemv(bits, q, s, x)[0], oracle.gemv(8, q, s, x)[0])
    with pytest.raises(ValueError):
        oracle.gemv(bits, np.full((N, K), RANGE[bits], np.int8), s, x)


def test_generator_ranges():
    for bits in (5, 6):
        q = synth.weights(bits, 0, 11, 256, 0, 64)
        assert q.min() == -RANGE[bits] and q.max() == RANGE[bits] - 1


def test_widths_in_the_decode_stream():
    ts = workloads.decode_stream(fused=True)
    for bits in (5, 6):
        wt = workloads.as_width(ts, bits)
        q4_bytes = sum(t.bytes for t in ts if t.bits == 4)
        # q4 holds 9/16 byte per weight, q5 / q6 (9 + 2 (bits - 4)) / 16
        assert workloads.total_bytes(wt) - workloads.total_bytes(ts) == q4_bytes * 2 * (bits - 4) // 9


# ---------------------------------------------------------------- GPU
def _torch():
    import torch

    return torch


def _dev(a):
    torch = _torch()
    a = np.ascontiguousarray(a)
    return torch.from_numpy(a.view(np.uint8).ravel().copy()).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("bits", [5, 6])
@pytest.mark.parametrize("N,K", [(70, 192), (4099, 5120), (1, 64)])
def test_device_pack_and_register_decode(q4, cuda_device, bits, N, K):
    """The device packer writes the host packer's bytes; the debug decoder,
    through the kernels' fp16 and bf16 register decodes, returns every code
    bit-exactly (and both decodes agree)."""
    torch = _torch()
    q, s = synth.tensor(bits, 1, 71, N, K)
    host = q4.q4_pack_weights(bits, q, s, N, K)
    out = torch.full((host.size,), 0xAB, dtype=torch.uint8, device="cuda")
    q4.q4_pack_weights_device(bits, _dev(q), _dev(s).view(torch.int16), N, K, out)
    qo = torch.zeros(N * K, dtype=torch.int8, device="cuda")
    so = torch.zeros(N * (K // 32), dtype=torch.int16, device="cuda")
    q4.q4_unpack_device(bits, out, N, K, qo, so)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), host)
    assert np.array_equal(qo.cpu().numpy().reshape(N, K), q)
    assert np.array_equal(so.cpu().numpy().view(np.uint16).reshape(N, K // 32), s)


def _stack(q4, specs, M, xs, flags=None):
    torch = _torch()
    import gpu_helpers as H

    entries, out = [], []
    for bits, N, K, tid in specs:
        if bits == workloads.NVFP4:
            c, sc, t = synth.nvfp4_tensor(4, tid, N, K)
            q, s = (c, sc, t), None
            buf = torch.from_numpy(q4.q4_pack_nvfp4(c, sc, t, N, K)).cuda()
        else:
            q, s = synth.tensor(bits, 4, tid, N, K)
            buf = torch.from_numpy(q4.q4_pack_weights(bits, q, s, N, K)).cuda()
        y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
        entries.append((bits, N, K, buf, xs[K][1], y))
        out.append((bits, N, K, q, s, y))
    st = q4.layer_stack_create(entries, M, q4.Q4_STACK_INDEPENDENT if flags is None else flags)
    return st, out


WIDE_STACKS = {
    "q5": [(5, 1000, 5120, 81), (5, 17, 17408, 82), (5, 4099, 5120, 83), (5, 64, 256, 84)],
    "q6": [(6, 1000, 5120, 85), (6, 33, 256, 86), (6, 7168, 5120, 87)],
    # every format in one list (q4, q8, q5, q6, NVFP4 share the activations)
    "mixed": [(4, 1000, 5120, 88), (5, 3, 5120, 89), (8, 37, 5120, 90), (6, 2050, 5120, 91),
              (workloads.NVFP4, 96, 5120, 92), (5, 64, 256, 93)],
    # K = 128: stages of two chunks
    "su2": [(5, 100, 128, 94), (6, 40, 128, 95), (4, 2050, 5120, 96)],
}


def _check(out, xs, M):
    import gpu_helpers as H
    from oracle import nvfp4 as ON

    for bits, N, K, q, s, y in out:
        yy = y.cpu().numpy().reshape(M, N)
        assert np.all(np.isfinite(yy))
        if bits == workloads.NVFP4:
            y_ref, B = ON.gemv(*q, xs[K][0])
            ok, _, _ = oracle.within_tolerance(yy, y_ref, B)
            assert ok.all(), "NVFP4 product outside the tolerance"
            continue
        H.assert_parity(yy, q, s, xs[K][0], bits)


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("which", sorted(WIDE_STACKS))
def test_stream_stack_parity(q4, cuda_device, which, M):
    torch = _torch()
    import gpu_helpers as H

    specs = WIDE_STACKS[which]
    xs = {}
    for K in sorted({k for _, _, k, _ in specs}):
        x = synth.activations(4, synth.act_stream(K), M, K)
        xs[K] = (x, H.to_device_x(x))
    st, out = _stack(q4, specs, M, xs)
    assert st.launches() == 2
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    first = [y.cpu().numpy().copy() for *_, y in out]
    _check(out, xs, M)
    for *_, y in out:
        y.fill_(float("nan"))
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    for f, (*_, y) in zip(first, out):
        assert np.array_equal(y.cpu().numpy(), f)
    st.close()


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["wide_range", "huge", "tiny", "zeros"])
@pytest.mark.parametrize("M", [1, 4])
def test_activation_ranges(q4, cuda_device, case, M):
    torch = _torch()
    import gpu_helpers as H

    K = 5120
    x = synth.activations(6, synth.act_stream(46), M, K)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if case == "wide_range":
        xf[:, ::7] *= 2.0 ** 60
        xf[:, 3::11] *= 2.0 ** -60
    elif case == "tiny":
        xf *= 2.0 ** -100
    elif case == "huge":
        xf *= 2.0 ** 100
    else:
        xf[:] = 0.0
    x = synth.f64_to_bf16_bits(xf.ravel()).reshape(M, K)
    xs = {K: (x, H.to_device_x(x))}
    st, out = _stack(q4, [(5, 160, K, 97), (6, 96, K, 98), (4, 64, K, 99)], M, xs)
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    if case == "zeros":
        for *_, y in out:
            assert np.all(y.cpu().numpy() == 0.0)
    _check(out, xs, M)
    st.close()


@pytest.mark.gpu
@pytest.mark.parametrize("bits", [5, 6])
@pytest.mark.parametrize("M", [1, 3])
def test_degenerate_and_extreme_rows(q4, cuda_device, bits, M):
    """All-zero rows, rows of the extreme codes, a single nonzero code."""
    torch = _torch()
    import gpu_helpers as H

    N, K = 96, 5120
    r = RANGE[bits]
    q, s = synth.tensor(bits, 5, 100 + bits, N, K)
    q = q.copy()
    q[0::4] = 0
    q[1::4] = -r
    q[2::4] = r - 1
    q[3::8] = 0
    q[3::8, 1234] = -r
    x = synth.activations(5, synth.act_stream(47), M, K)
    y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
    buf = torch.from_numpy(q4.q4_pack_weights(bits, q, s, N, K)).cuda()
    st = q4.layer_stack_create([(bits, N, K, buf, H.to_device_x(x), y)], M, q4.Q4_STACK_INDEPENDENT)
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    yy = y.cpu().numpy().reshape(M, N)
    assert np.all(yy[:, 0::4] == 0)
    H.assert_parity(yy, q, s, x, bits)
    st.close()


@pytest.mark.gpu
def test_unsupported_modes_are_refused(q4, cuda_device):
    torch = _torch()
    import gpu_helpers as H

    N, K = 64, 256
    q, s = synth.tensor(5, 1, 101, N, K)
    p = torch.from_numpy(q4.q4_pack_weights(5, q, s, N, K)).cuda()
    x = H.to_device_x(synth.activations(1, 1, 1, K))
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    for flags in (0, q4.Q4_STACK_GRAPH):
        with pytest.raises(q4.Q4Error, match="UNSUPPORTED"):
            q4.layer_stack_create([(5, N, K, p, x, y)], 1, flags)


@pytest.mark.gpu
@pytest.mark.parametrize("bits,M", [(5, 1), (6, 1), (6, 4)])
def test_full_decode_stream_at_other_widths_sampled(q4, cuda_device, bits, M):
    """The 64-layer decode stream with its q4 tensors at 5 or 6 bits (16.3 /
    18.8 GB) in one stream-mode launch; sampled rows against the oracle."""
    torch = _torch()
    import gpu_helpers as H

    tensors = workloads.as_width(workloads.decode_stream(fused=True), bits)
    st = workloads.DeviceStream(tensors, M, flags=q4.Q4_STACK_INDEPENDENT)
    assert st.stack.launches() == 2
    st.run()
    st.check()
    torch.cuda.synchronize()
    rng = np.random.default_rng(bits * 10 + M)
    for i in [0, 1, 2, 3, 12, 13, 14, 15, 128, 254, 255, 256]:
        t = tensors[i]
        y = st.y[i].cpu().numpy().reshape(M, t.N)
        assert np.all(np.isfinite(y)), t.name
        x = synth.activations(st.seed, synth.act_stream(workloads.activation_stream_id(t.K)), M, t.K)
        for r in sorted({0, t.N - 1} | set(rng.integers(0, t.N, 6).tolist())):
            q, s = synth.tensor(t.bits, st.seed, t.tensor_id, t.N, t.K, row0=r, nrows=1)
            H.assert_parity(y[:, r:r + 1], q, s, x, t.bits)
    st.close()
    torch.cuda.empty_cache()

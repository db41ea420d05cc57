"""The dependent decode chain: the oracle's steps pinned by closed forms and
identities (CPU); each step kernel against the oracle, the captured chain
against the same steps called one by one, and every op of the two-layer and
of the 64-layer chain, in both chain forms, against the oracle element by
element on the GPU's own inputs (GPU)."""
import numpy as np
import pytest

from oracle import chain as OC
import oracle
import chain_check
from bit_weight_gemv_q4_b200 import synth, workloads

SMALL = workloads.ChainShape(layers=2, hidden=1024, ffn=2048, kv=256, vocab=4096)


# ---------------------------------------------------------------- oracle pins
def test_bf16_rounding_hand_values():
    vals = np.array([1.0, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -2.5, 2.0 ** -130, 0.0, 1 + 2.0 ** -8 + 2.0 ** -30])
    # ties go to the even mantissa: 1 + 2^-8 -> 1.0, 1 + 3*2^-8 -> 1 + 2^-6; the subnormal 2^-130 is 8 * 2^-133;
    # just above the tie rounds up
    assert OC.bf16_exact(vals).tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0008, 0x0000, 0x3F81]
    # the two-step conversion (fp64 -> fp32 -> bf16) differs from the one-step
    # rounding only where the fp32 value lands exactly on a bf16 tie
    z = np.random.default_rng(1).normal(0, 3, 20000)
    d = OC.bf16_exact(z) != OC.bf16_bits(z)
    f32 = z.astype(np.float32).view(np.uint32)
    assert np.all((f32[d] & 0xFFFF) == 0x8000)


def test_silu_identities():
    z = np.linspace(-30, 30, 601)
    assert np.allclose(OC.silu(z) - OC.silu(-z), z, rtol=0, atol=1e-12)  # silu(z) - silu(-z) = z
    assert OC.silu(np.array([0.0]))[0] == 0.0
    assert abs(OC.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(OC.silu(np.array([1.0]))[0] - 1.0 / (1.0 + np.exp(-1.0))) < 1e-16


def test_rmsnorm_closed_forms():
    c = np.full((1, 512), 3.0)
    h, z = OC.residual_rmsnorm(None, c, None)
    assert np.array_equal(h, c)
    assert np.allclose(z, 3.0 / np.sqrt(9.0 + OC.EPS), rtol=0, atol=1e-15)
    rng = np.random.default_rng(2)
    h0, y = rng.normal(0, 2, (3, 256)), rng.normal(0, 2, (3, 256))
    g = 1 + rng.normal(0, 0.1, 256)
    h1, z = OC.residual_rmsnorm(h0, y, g)
    assert np.allclose(h1, h0 + y, rtol=0, atol=1e-15)
    zn = z / g  # mean square of the normalised rows is ms / (ms + eps)
    ms = np.mean(h1 * h1, axis=1)
    assert np.allclose(np.mean(zn * zn, axis=1), ms / (ms + OC.EPS), rtol=1e-12)
    # invariant under scaling when eps is negligible against the mean square
    _, z2 = OC.residual_rmsnorm(None, (h0 + y) * 1e3, g)
    assert np.allclose(z, z2, rtol=1e-6)


def test_swiglu_closed_forms():
    y = np.zeros((2, 8))
    y[0, :4] = [0.0, 1.0, -1.0, 40.0]
    y[0, 4:] = [5.0, 0.0, 2.0, 0.5]
    z = OC.swiglu(y, 4)
    assert z[0, 0] == 0.0 and z[0, 1] == 0.0
    assert np.isclose(z[0, 2], -1.0 / (1.0 + np.e) * 2.0)
    assert np.isclose(z[0, 3], 40.0 * 0.5)
    assert not z[1].any()


def test_near_tie_window():
    t = np.array([1 + 2.0 ** -8, 1.0, 1 + 2.0 ** -8 + 2.0 ** -20])
    assert OC.near_bf16_tie(t, 0.0).tolist() == [True, False, False]
    assert OC.near_bf16_tie(t, 2.0 ** -18).tolist() == [True, False, True]


def test_chain_shape_of_the_decode_stream():
    assert workloads.chain_tensors(workloads.ChainShape()) == workloads.decode_stream(fused=True)


def test_chain_shapes_meet_the_one_launch_conditions():
    """The conditions include/q4gemv.h states for Q4_CHAIN_PERSISTENT hold for
    the decode chain and the small one at every M: stages of four chunks at
    M <= 2 and of two at M >= 3 (q4 K a multiple of 256 / 128, q8 K of 128 /
    64), step rows N % 8 == 0, and the rings, the activation buffer (M rows
    of the largest K or step row, bf16) and the per-warp tile scratch within
    227 KB of shared memory less 1 KB."""
    for shape in (workloads.ChainShape(), SMALL):
        tensors = workloads.chain_tensors(shape)
        assert shape.hidden % 8 == 0 and shape.ffn % 8 == 0
        for M in (1, 2, 3, 4):
            su = 4 if M <= 2 else 2
            for t in tensors:
                assert t.bits in (4, 8) and t.N > 0
                assert t.K % (su * (64 if t.bits == 4 else 32)) == 0, t.name
            x_max = max(max(t.K for t in tensors), shape.hidden, shape.ffn)
            rings = -(-(16 * 2 * su * 1152 + 16 * 2 * 8) // 128) * 128  # 16 warps x 2 stages, barriers
            x_bytes = -(-2 * M * x_max // 128) * 128
            assert rings + x_bytes + 16 * M * 32 * 4 <= 227 * 1024 - 1024, (M, rings, x_bytes)


# ---------------------------------------------------------------- oracle chain
def oracle_chain(shape, M, seed):
    """Every intermediate of the chain from the oracle alone (inputs from the
    seeded generator): dict with x (bf16 bits), z (pre-rounding), y, B."""
    H, F, L = shape.hidden, shape.ffn, shape.layers
    tensors = workloads.chain_tensors(shape)
    gam = OC.bf16_value(workloads.chain_gammas(shape, seed))
    emb = OC.bf16_value(synth.activations(seed, workloads.chain_input_stream(0), M, H))
    out = {"x": {}, "z": {}, "y": {}, "B": {}}

    def prod(i, xbits):
        t = tensors[i]
        q, s = synth.tensor(t.bits, seed, t.tensor_id, t.N, t.K)
        y, B = OC.product(t.bits, q, s, xbits)
        out["y"][i], out["B"][i] = y, B
        return y

    h = None
    y_prev = emb
    for layer in range(L):
        h, z = OC.residual_rmsnorm(h, y_prev, gam[2 * layer])
        x = OC.bf16_exact(z)
        out["z"][("qkv", layer)], out["x"][("qkv", layer)] = z, x
        prod(4 * layer, x)
        xm = synth.activations(seed, workloads.chain_input_stream(1 + layer), M, H)
        y_o = prod(4 * layer + 1, xm)
        h, z = OC.residual_rmsnorm(h, y_o, gam[2 * layer + 1])
        x = OC.bf16_exact(z)
        out["z"][("gu", layer)], out["x"][("gu", layer)] = z, x
        y_gu = prod(4 * layer + 2, x)
        z = OC.swiglu(y_gu, F)
        x = OC.bf16_exact(z)
        out["z"][("down", layer)], out["x"][("down", layer)] = z, x
        y_prev = prod(4 * layer + 3, x)
    h, z = OC.residual_rmsnorm(h, y_prev, gam[2 * L])
    x = OC.bf16_exact(z)
    out["z"][("head", L)], out["x"][("head", L)] = z, x
    prod(4 * L, x)
    out["h"] = h
    return out


# ---------------------------------------------------------------- GPU
def _torch():
    import torch

    return torch


def _f32(host):
    return _torch().from_numpy(np.ascontiguousarray(host, dtype=np.float32)).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("set_", [False, True])
def test_rmsnorm_kernel_matches_the_oracle(cuda_device, M, set_):
    """bf16 outputs equal the oracle's except within 2^-17 (relative) of a
    rounding tie, where the fp32 computation may round either way; h is the
    fp32 sum."""
    import bit_weight_gemv_q4_b200 as q4

    torch = _torch()
    N = 5120
    h0 = synth.normals_f64(3, 900, 0, M * N).astype(np.float32).reshape(M, N) * 4
    y = synth.normals_f64(3, 901, 0, M * N).astype(np.float32).reshape(M, N) * 7
    g = synth.f64_to_bf16_bits(1 + synth.normals_f64(3, 902, 0, N) / 16)
    hd, yd = _f32(h0), _f32(y)
    gd = torch.from_numpy(g.view(np.int16)).cuda()
    xd = torch.empty(M * N, dtype=torch.int16, device="cuda")
    q4.q4_residual_rmsnorm(hd, yd, gd, xd, N, M, set_)
    torch.cuda.synchronize()
    h_ref, z = OC.residual_rmsnorm(None if set_ else h0.astype(np.float64), y.astype(np.float64), OC.bf16_value(g))
    assert np.array_equal(hd.cpu().numpy().reshape(M, N), (y if set_ else h0 + y).astype(np.float32))
    x = xd.cpu().numpy().view(np.uint16).reshape(M, N)
    diff = x != OC.bf16_exact(z)
    assert not (diff & ~OC.near_bf16_tie(z, 2.0 ** -17)).any()
    assert diff.mean() < 1e-3


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 3])
def test_swiglu_kernel_matches_the_oracle(cuda_device, M):
    import bit_weight_gemv_q4_b200 as q4

    torch = _torch()
    N = 17408
    y = (synth.normals_f64(4, 903, 0, M * 2 * N) * 6).astype(np.float32).reshape(M, 2 * N)
    xd = torch.empty(M * N, dtype=torch.int16, device="cuda")
    q4.q4_swiglu(_f32(y), xd, N, M)
    torch.cuda.synchronize()
    z = OC.swiglu(y.astype(np.float64), N)
    x = xd.cpu().numpy().view(np.uint16).reshape(M, N)
    diff = x != OC.bf16_exact(z)
    assert not (diff & ~OC.near_bf16_tie(z, 2.0 ** -19)).any()
    assert diff.mean() < 1e-3


def _outputs(ch):
    torch = _torch()
    torch.cuda.synchronize()
    got = {"y": [y.cpu().numpy().copy() for y in ch.w.y]}
    got["x"] = [t.cpu().numpy().copy() for t in ch.x_qkv + ch.x_gu + ch.x_down + [ch.x_head]]
    got["h"] = ch.h.cpu().numpy().copy()
    return got


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 4])
def test_chain_equals_its_steps_called_one_by_one(cuda_device, M):
    """The captured chain (with and without programmatic dependent launch) is
    bitwise the sequence of single calls on the same buffers."""
    import bit_weight_gemv_q4_b200 as q4

    torch = _torch()
    ch = workloads.DeviceChain(SMALL, M, seed=5, flags=q4.Q4_CHAIN_GRAPH)
    assert ch.stack.launches() == 7 * SMALL.layers + 2
    ch.run()
    ch.check()
    graph = _outputs(ch)
    ch.run()
    again = _outputs(ch)
    assert all(np.array_equal(a, b) for a, b in zip(graph["y"] + graph["x"], again["y"] + again["x"]))
    nopdl = q4.layer_chain_create(ch.ops, M, q4.Q4_STACK_NO_PDL)
    q4.layer_stack_run(nopdl)
    q4.layer_stack_check(nopdl)
    third = _outputs(ch)
    assert all(np.array_equal(a, b) for a, b in zip(graph["y"] + graph["x"], third["y"] + third["x"]))
    nopdl.close()
    # the same ops, one call each
    for y in ch.w.y:
        y.fill_(float("nan"))
    ws = torch.zeros(max(q4.q4_gemv_workspace_bytes(t.bits, t.N, t.K, M) for t in ch.w.tensors), dtype=torch.uint8,
                     device="cuda")
    for kind, bits, N, K, packed, inp, out, resid in ch.ops:
        if kind == q4.Q4_OP_PRODUCT:
            (q4.q4_gemv if bits == 4 else q4.q8_gemv)(packed, N, K, inp, M, out, ws)
        elif kind == q4.Q4_OP_RESIDUAL_RMSNORM:
            q4.q4_residual_rmsnorm(resid, inp, packed, out, N, M, bits == 1)
        else:
            q4.q4_swiglu(inp, out, N, M)
    q4.q4_workspace_check(ws)
    single = _outputs(ch)
    assert all(np.array_equal(a, b) for a, b in zip(graph["y"] + graph["x"], single["y"] + single["x"]))
    assert np.array_equal(graph["h"], single["h"])
    ch.close()


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["graph", "persistent"])
@pytest.mark.parametrize("M", [1, 2, 4])
def test_chain_ops_against_the_oracle(cuda_device, M, mode):
    """Every op of the two-layer chain on the GPU's own inputs: every output
    of every product within the product tolerance, every activation of every
    step equal to the oracle's outside the rounding-tie window, the residual
    stream equal to its fp32 replay.  The first activations (the norm of the
    embedding) also equal those of the oracle's own chain, computed from the
    seeded inputs alone."""
    import bit_weight_gemv_q4_b200 as q4

    ch = workloads.DeviceChain(SMALL, M, seed=6,
                               flags=q4.Q4_CHAIN_PERSISTENT if mode == "persistent" else q4.Q4_CHAIN_GRAPH)
    ch.run()
    ch.check()
    stats = chain_check.check(ch)
    assert stats["products"] == 4 * SMALL.layers + 1 and stats["norms"] == 2 * SMALL.layers + 1
    assert stats["tie_diffs"] <= 1e-3 * stats["values"]
    ref = oracle_chain(SMALL, M, 6)
    x0 = ch.x_qkv[0].cpu().numpy().view(np.uint16).reshape(M, SMALL.hidden)
    diff = x0 != ref["x"][("qkv", 0)]
    assert not (diff & ~OC.near_bf16_tie(ref["z"][("qkv", 0)], 2.0 ** -17)).any()
    ch.close()


# ---------------------------------------------------------- the one-launch chain
@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 2])
def test_persistent_chain_equals_its_ops_called_one_by_one(cuda_device, M):
    """The chain as one cooperative launch is bitwise the same ops run one
    call at a time on the same buffers: each product as a one-product
    stream-mode stack (the same split and decode: stages of four chunks at
    M <= 2), each step as q4_residual_rmsnorm / q4_swiglu (the same sum of
    squares); and two runs agree bitwise."""
    import bit_weight_gemv_q4_b200 as q4

    torch = _torch()
    ch = workloads.DeviceChain(SMALL, M, seed=7, flags=q4.Q4_CHAIN_PERSISTENT)
    assert ch.stack.launches() == 1
    ch.run()
    ch.check()
    one = _outputs(ch)
    ch.run()
    ch.check()
    again = _outputs(ch)
    for key in ("y", "x"):
        assert all(np.array_equal(a, b) for a, b in zip(one[key], again[key]))
    assert np.array_equal(one["h"], again["h"])
    for y in ch.w.y:
        y.fill_(float("nan"))
    for x in ch.x_qkv + ch.x_gu + ch.x_down + [ch.x_head]:
        x.fill_(-1)
    ch.h.fill_(float("nan"))
    for kind, bits, N, K, packed, inp, out, resid in ch.ops:
        if kind == q4.Q4_OP_PRODUCT:
            st = q4.layer_stack_create([(bits, N, K, packed, inp, out)], M, q4.Q4_STACK_INDEPENDENT)
            q4.layer_stack_run(st)
            q4.layer_stack_check(st)
            st.close()
        elif kind == q4.Q4_OP_RESIDUAL_RMSNORM:
            q4.q4_residual_rmsnorm(resid, inp, packed, out, N, M, bits == 1)
        else:
            q4.q4_swiglu(inp, out, N, M)
    torch.cuda.synchronize()
    single = _outputs(ch)
    for i, (a, b) in enumerate(zip(one["y"], single["y"])):
        assert np.array_equal(a, b), workloads.chain_tensors(SMALL)[i].name
    for a, b in zip(one["x"], single["x"]):
        assert np.array_equal(a, b)
    assert np.array_equal(one["h"], single["h"])
    ch.close()


@pytest.mark.gpu
@pytest.mark.parametrize("M", [1, 4])
def test_full_chain_ops_against_the_oracle(cuda_device, M):
    """The 64-layer chain with the output head, captured (one kernel per op)
    and as one launch: both reproducible bitwise run to run, and every op of
    each checked on that run's own inputs: 16 rows of every product
    (including the 248,320-row head) within the product tolerance, every
    activation of every step outside the rounding-tie window, the final
    residual stream equal to its fp32 replay."""
    import bit_weight_gemv_q4_b200 as q4

    torch = _torch()
    ch = workloads.DeviceChain(workloads.ChainShape(), M, flags=q4.Q4_CHAIN_GRAPH)
    assert ch.stack.launches() == 64 * 7 + 2
    persistent = q4.layer_chain_create(ch.ops, M, q4.Q4_CHAIN_PERSISTENT)
    assert persistent.launches() == 1
    try:
        for name, stack in (("graph", ch.stack), ("persistent", persistent)):
            q4.layer_stack_run(stack)
            q4.layer_stack_check(stack)
            a = ch.logits.cpu().numpy().copy()
            q4.layer_stack_run(stack)
            q4.layer_stack_check(stack)
            assert np.all(np.isfinite(a)) and np.array_equal(a, ch.logits.cpu().numpy()), name
            stats = chain_check.check(ch, sample_rows=16)
            assert stats["products"] == 257 and stats["norms"] == 129 and stats["swiglus"] == 64, name
            assert stats["tie_diffs"] <= 1e-3 * stats["values"], name
    finally:
        persistent.close()
        ch.close()
        torch.cuda.empty_cache()


@pytest.mark.gpu
def test_chain_form_chosen_by_default(cuda_device):
    """Without a form named, the chain runs as the graph at every M; naming
    both forms is an argument error."""
    import bit_weight_gemv_q4_b200 as q4

    for M, launches in ((1, 7 * SMALL.layers + 2), (2, 7 * SMALL.layers + 2)):
        ch = workloads.DeviceChain(SMALL, M, seed=9)
        assert ch.stack.launches() == launches
        ch.close()
    ch = workloads.DeviceChain(SMALL, 1, seed=9, flags=q4.Q4_CHAIN_GRAPH)
    with pytest.raises(q4.Q4Error) as e:
        q4.layer_chain_create(ch.ops, 1, q4.Q4_CHAIN_PERSISTENT | q4.Q4_CHAIN_GRAPH)
    assert e.value.code == q4.Q4_ERR_INVALID_ARG
    ch.close()


@pytest.mark.gpu
def test_persistent_chain_rejects_what_it_cannot_order(cuda_device):
    import bit_weight_gemv_q4_b200 as q4

    torch = _torch()
    ch = workloads.DeviceChain(SMALL, 1, seed=8)
    P = q4.Q4_CHAIN_PERSISTENT
    # two ops writing one buffer
    ops = list(ch.ops)
    k = next(i for i, op in enumerate(ops) if op[0] == q4.Q4_OP_PRODUCT)
    k2 = next(i for i, op in enumerate(ops) if op[0] == q4.Q4_OP_PRODUCT and i > k)
    op2 = list(ops[k2])
    op2[6] = ops[k][6]
    bad = ops[:k2] + [tuple(op2)] + ops[k2 + 1:]
    with pytest.raises(q4.Q4Error) as e:
        q4.layer_chain_create(bad, 1, P)
    assert e.value.code == q4.Q4_ERR_UNSUPPORTED
    # a q4 product whose K is not a multiple of 256
    w = torch.zeros(q4.q4_packed_bytes(4, 32, 96), dtype=torch.uint8, device="cuda")
    x = torch.zeros(96, dtype=torch.int16, device="cuda")
    y = torch.zeros(32, dtype=torch.float32, device="cuda")
    with pytest.raises(q4.Q4Error) as e:
        q4.layer_chain_create([(q4.Q4_OP_PRODUCT, 4, 32, 96, w, x, y, None)], 1, P)
    assert e.value.code == q4.Q4_ERR_UNSUPPORTED
    # at M = 4 (stages of two chunks) a q4 K must be a multiple of 128
    y4 = torch.zeros(4 * 32, dtype=torch.float32, device="cuda")
    for K, ok in ((192, False), (256, True)):
        w = torch.zeros(q4.q4_packed_bytes(4, 32, K), dtype=torch.uint8, device="cuda")
        x = torch.zeros(4 * K, dtype=torch.int16, device="cuda")
        if ok:
            q4.layer_chain_create([(q4.Q4_OP_PRODUCT, 4, 32, K, w, x, y4, None)], 4, P).close()
        else:
            with pytest.raises(q4.Q4Error) as e:
                q4.layer_chain_create([(q4.Q4_OP_PRODUCT, 4, 32, K, w, x, y4, None)], 4, P)
            assert e.value.code == q4.Q4_ERR_UNSUPPORTED
    ch.close()


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["wide_range", "huge", "zeros"])
def test_persistent_chain_activation_ranges(cuda_device, case):
    """Products of the one-launch chain on activations staged from global
    memory: beyond fp16's range after any power-of-two scaling (the bf16
    decode), far above it (scaled in exactly), all zero.  The second product
    reads the same activations and takes them from shared memory without
    staging them again.  Each output is within the tolerance of the oracle
    and bitwise the one-product stream-mode stack's."""
    import bit_weight_gemv_q4_b200 as q4
    import gpu_helpers as H

    torch = _torch()
    K = 5120
    x = synth.activations(6, synth.act_stream(44), 1, K)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if case == "wide_range":
        xf[:, ::7] *= 2.0 ** 60
        xf[:, 3::11] *= 2.0 ** -60
    elif case == "huge":
        xf *= 2.0 ** 100
    else:
        xf[:] = 0.0
    x = synth.f64_to_bf16_bits(xf.ravel()).reshape(1, K)
    x_dev = H.to_device_x(x)
    ops, hosts, ys = [], [], []
    for bits, N, tid in ((4, 160, 53), (8, 96, 54)):
        q, s = synth.tensor(bits, 6, tid, N, K)
        packed = H.to_device_packed(bits, q, s, N, K)
        y = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
        ops.append((q4.Q4_OP_PRODUCT, bits, N, K, packed, x_dev, y, None))
        hosts.append((bits, N, q, s, packed))
        ys.append(y)
    ch = q4.layer_chain_create(ops, 1, q4.Q4_CHAIN_PERSISTENT)
    q4.layer_stack_run(ch)
    q4.layer_stack_check(ch)
    torch.cuda.synchronize()
    for (bits, N, q, s, packed), y in zip(hosts, ys):
        yy = y.cpu().numpy().reshape(1, N).copy()
        if case == "zeros":
            assert np.all(yy == 0.0)
        H.assert_parity(yy, q, s, x, bits)
        y2 = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
        st = q4.layer_stack_create([(bits, N, K, packed, x_dev, y2)], 1, q4.Q4_STACK_INDEPENDENT)
        q4.layer_stack_run(st)
        q4.layer_stack_check(st)
        assert np.array_equal(yy.ravel(), y2.cpu().numpy())
        st.close()
    ch.close()

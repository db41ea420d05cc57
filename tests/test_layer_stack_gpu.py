"""The captured layer stack: same results as one call per product, oracle parity,
and the full 64-layer decode stream (13.7 GB) checked on sampled rows and, in
every mode, on every output."""
import numpy as np
import pytest

import oracle

from bit_weight_gemv_q4_b200 import synth, workloads
from bit_weight_gemv_q4_b200.workloads import Tensor
import gpu_helpers as H

pytestmark = pytest.mark.gpu

# every product has an even number of chunks per tile and whole q4 chunks:
# eligible for both persistent modes
MIXED = [
    Tensor("a", 4, 1000, 5120, 201), Tensor("b", 8, 37, 128, 202), Tensor("c", 4, 17, 17408, 203),
    Tensor("d", 8, 4099, 5120, 204), Tensor("e", 4, 64, 128, 205), Tensor("f", 4, 7168, 5120, 206),
]
# every product's chunks per tile a multiple of 4: stream mode with stages of
# four chunks (MIXED, with a q4 K of 128 = 2 chunks, uses stages of two)
MIXED4 = [
    Tensor("a4", 4, 1000, 5120, 221), Tensor("b4", 8, 37, 128, 222), Tensor("c4", 4, 17, 17408, 223),
    Tensor("d4", 8, 4099, 5120, 224), Tensor("e4", 4, 64, 256, 225), Tensor("f4", 4, 7168, 5120, 226),
    Tensor("g4", 8, 3, 256, 227),
]
# a q4 K that is an odd multiple of 32 (even chunk count): ordered persistent
# mode, also when stream mode is asked for
HALF = [Tensor("j", 4, 64, 96, 210), Tensor("k", 8, 100, 5120, 211)]
# odd chunk counts per tile: graph mode only
ODD = [Tensor("g", 8, 37, 96, 207), Tensor("h", 4, 64, 4096 + 32, 208), Tensor("i", 4, 300, 5120, 209)]


@pytest.fixture(scope="module")
def q4(cuda_device):
    import bit_weight_gemv_q4_b200 as lib

    return lib


def _y(stream, i):
    t = stream.tensors[i]
    return stream.y[i].cpu().numpy().reshape(stream.M, t.N)


def _host_rows(stream, i, r0, n):
    t = stream.tensors[i]
    q, s = synth.tensor(t.bits, stream.seed, t.tensor_id, t.N, t.K, row0=r0, nrows=n)
    x = synth.activations(stream.seed, synth.act_stream(workloads.activation_stream_id(t.K)), stream.M, t.K)
    return q, s, x


def _check_stack(q4, tensors, M, flags, expect_launches):
    torch = H.torch()
    st = workloads.DeviceStream(tensors, M, flags=flags)
    assert st.stack.launches() == expect_launches
    st.run()
    st.check()
    first = [_y(st, i).copy() for i in range(len(tensors))]
    # a second run is bitwise identical
    for y in st.y:
        y.fill_(float("nan"))
    st.run()
    st.check()
    for i in range(len(tensors)):
        assert np.array_equal(_y(st, i), first[i])
    # each product equals a direct call on the same device buffers
    for i, t in enumerate(tensors):
        ws = H.workspace(t.bits, t.N, t.K, M)
        y = torch.empty(M * t.N, device="cuda")
        (q4.q4_gemv if t.bits == 4 else q4.q8_gemv)(st.packed[i], t.N, t.K, st.x[t.K], M, y, ws)
        q4.q4_workspace_check(ws)
        assert np.array_equal(y.cpu().numpy().reshape(M, t.N), first[i]), t.name
    # and the oracle, on every row
    for i, t in enumerate(tensors):
        q, s, x = _host_rows(st, i, 0, t.N)
        H.assert_parity(first[i], q, s, x, t.bits)
    st.close()
    return first


@pytest.mark.parametrize("M", [1, 4])
def test_stack_modes_equal_single_calls_and_oracle(q4, M):
    persistent = _check_stack(q4, MIXED, M, q4.Q4_STACK_ORDERED, 1)
    graph = _check_stack(q4, MIXED, M, q4.Q4_STACK_GRAPH, len(MIXED))
    nopdl = _check_stack(q4, MIXED, M, q4.Q4_STACK_NO_PDL, len(MIXED))
    for a, b, c in zip(persistent, graph, nopdl):
        assert np.array_equal(a, b) and np.array_equal(a, c)


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("tensors", [MIXED, MIXED4], ids=["stages2", "stages4"])
def test_stream_mode_of_independent_products(q4, M, tensors):
    """Stream mode splits the concatenated products between warps differently
    from one call per product: the outputs are compared with the oracle (every
    row) and with single calls within the product tolerance, and two runs are
    bitwise identical."""
    torch = H.torch()
    st = workloads.DeviceStream(tensors, M, flags=q4.Q4_STACK_INDEPENDENT)
    # activation preparation + one stream kernel per group: at M = 1 one group
    # (every activation resident); with stages of four chunks at M >= 2 the
    # products are grouped so that each group's activations stay resident
    # (K 128 / 256 / 5120 together and K 17408 apart, resident at M = 2, with
    # its slices in the stages at M = 3 and 4; at M = 4 the q8 copy of the
    # 5120-value input needs a group of its own)
    expect = 2 if M == 1 or tensors is MIXED else {2: 3, 3: 3, 4: 4}[M]
    assert st.stack.launches() == expect
    st.run()
    st.check()
    first = [_y(st, i).copy() for i in range(len(tensors))]
    for y in st.y:
        y.fill_(float("nan"))
    st.run()
    st.check()
    for i, t in enumerate(tensors):
        assert np.array_equal(_y(st, i), first[i]), t.name
        q, s, x = _host_rows(st, i, 0, t.N)
        H.assert_parity(first[i], q, s, x, t.bits)
        ws = H.workspace(t.bits, t.N, t.K, M)
        y = torch.empty(M * t.N, device="cuda")
        (q4.q4_gemv if t.bits == 4 else q4.q8_gemv)(st.packed[i], t.N, t.K, st.x[t.K], M, y, ws)
        q4.q4_workspace_check(ws)
        import oracle
        _, B = oracle.gemv(t.bits, q, s, x)
        ok, _, _ = oracle.within_tolerance(first[i], y.cpu().numpy().reshape(M, t.N).astype(np.float64), B)
        assert ok.all(), t.name
    st.close()


@pytest.mark.parametrize("M", [1, 2])
def test_half_empty_chunks_fall_back_to_ordered_mode(q4, M):
    _check_stack(q4, HALF, M, q4.Q4_STACK_INDEPENDENT, 1)


@pytest.mark.parametrize("M", [1, 3])
def test_stack_with_odd_chunk_counts_uses_graph_mode(q4, M):
    _check_stack(q4, ODD, M, 0, len(ODD))


@pytest.mark.parametrize("M,mode", [(1, "ordered"), (4, "ordered"), (1, "stream"), (4, "stream")])
def test_full_decode_stream_sampled(q4, M, mode):
    """All 257 products of one decode step (64 layers + q8 head, 13.7 GB) in one
    persistent kernel; sampled rows of several tensors against the oracle."""
    torch = H.torch()
    tensors = workloads.decode_stream(fused=True)
    st = workloads.DeviceStream(tensors, M, flags=q4.Q4_STACK_ORDERED if mode == "ordered" else q4.Q4_STACK_INDEPENDENT)
    # one persistent kernel for the 257 products (stream mode: after xprep_kernel;
    # at M = 4 two groups, the products of the 5120- and the 17,408-value inputs)
    assert st.stack.launches() == (1 if mode == "ordered" else 2 if M == 1 else 3)
    st.run()
    st.run()
    st.check()
    torch.cuda.synchronize()
    rng = np.random.default_rng(M)
    pick = [0, 1, 2, 3, 12, 13, 14, 15, 128, 254, 255, 256]  # layer 0, layer 3 (q8 mixer), layer 32, last, head
    for i in pick:
        t = tensors[i]
        y = _y(st, i)
        rows = sorted({0, t.N - 1} | set(rng.integers(0, t.N, 6).tolist()))
        for r in rows:
            q, s, x = _host_rows(st, i, r, 1)
            H.assert_parity(y[:, r:r + 1], q, s, x, t.bits)
        assert np.all(np.isfinite(y)), t.name
    st.close()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("M", [1, 4])
def test_full_decode_stream_every_output(q4, M):
    """Every output of all 257 products of one decode step (64 layers + the
    248,320-row q8 head: 13.7 GB of weights), in stream, ordered and graph
    mode, within the product tolerance of the fp64 oracle, which is
    regenerated tensor by tensor on the host (13.7 GB of codes per M).  The
    modes split the products differently (stream mode: one stream-K range over
    all of them, across product boundaries), so this also covers every place a
    split falls at full size."""
    torch = H.torch()
    tensors = workloads.decode_stream(fused=True)
    st = workloads.DeviceStream(tensors, M, flags=q4.Q4_STACK_INDEPENDENT)
    got = {}
    for mode, flags in (("stream", None), ("ordered", q4.Q4_STACK_ORDERED), ("graph", q4.Q4_STACK_GRAPH)):
        stack = st.stack if flags is None else st.make_stack(flags)
        for y in st.y:
            y.fill_(float("nan"))
        q4.layer_stack_run(stack)
        q4.layer_stack_check(stack)
        torch.cuda.synchronize()
        got[mode] = [_y(st, i).copy() for i in range(len(tensors))]
        if flags is not None:
            stack.close()
    x = {K: synth.activations(st.seed, synth.act_stream(workloads.activation_stream_id(K)), M, K)
         for K in workloads.distinct_k(tensors)}
    st.close()
    torch.cuda.empty_cache()
    worst = 0.0
    for i, t in enumerate(tensors):
        q, s = synth.tensor(t.bits, 0, t.tensor_id, t.N, t.K)
        y_ref, B = oracle.gemv(t.bits, q, s, x[t.K])
        del q, s
        for mode, ys in got.items():
            ok, err, bound = oracle.within_tolerance(ys[i], y_ref, B)
            if not ok.all():
                m, r = np.argwhere(~ok)[0]
                raise AssertionError(f"{mode} {t.name}: {(~ok).sum()} of {ok.size} outside tolerance, first row {r} "
                                     f"m {m}: {ys[i][m, r]} vs {y_ref[m, r]}")
            worst = max(worst, float((err / np.maximum(B, 1e-30)).max()))
    print(f"M={M}: worst |y - y_ref| / sum|w x| over all outputs and modes: {worst:.3g}")


@pytest.mark.parametrize("mode", ["ordered", "stream", "graph"])
@pytest.mark.parametrize("M", [1, 3])
def test_degenerate_rows_in_stacks(q4, mode, M):
    """All-zero rows (nonzero scales), single-code rows and one-group rows in
    every stack mode: within the tolerance, which is 1e-6 on a zero row."""
    torch = H.torch()
    K = 5120
    specs = [(4, 96), (8, 64)]
    x = synth.activations(5, synth.act_stream(42), M, K)
    x_dev = H.to_device_x(x)
    entries, hosts, ys = [], [], []
    for bits, N in specs:
        q, s = H.degenerate_rows(bits, N, K, seed=bits)
        y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
        entries.append((bits, N, K, H.to_device_packed(bits, q, s, N, K), x_dev, y))
        hosts.append((q, s))
        ys.append(y)
    flags = {"ordered": q4.Q4_STACK_ORDERED, "stream": q4.Q4_STACK_INDEPENDENT, "graph": q4.Q4_STACK_GRAPH}[mode]
    st = q4.layer_stack_create(entries, M, flags)
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    for (bits, N), (q, s), y in zip(specs, hosts, ys):
        H.assert_parity(y.cpu().numpy().reshape(M, N), q, s, x, bits)
    st.close()


@pytest.mark.parametrize("case", ["wide_range", "tiny", "huge", "zeros", "subnormal"])
@pytest.mark.parametrize("M", [1, 4])
def test_stream_mode_activation_ranges(q4, case, M):
    """Activations that fp16 cannot hold after any power-of-two scaling (a
    dynamic range beyond 2^40: the bf16 fallback), activations far below or
    above fp16's range (scaled into it exactly), all-zero activations and
    bf16 subnormals: every product within the tolerance."""
    torch = H.torch()
    K = 5120
    x = synth.activations(6, synth.act_stream(43), M, K)
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
        xf *= 2.0 ** -128  # many elements become bf16 subnormals
    x = synth.f64_to_bf16_bits(xf.ravel()).reshape(M, K)
    x_dev = H.to_device_x(x)
    entries, hosts, ys = [], [], []
    for bits, N, tid in ((4, 160, 51), (8, 96, 52)):
        q, s = synth.tensor(bits, 6, tid, N, K)
        y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
        entries.append((bits, N, K, H.to_device_packed(bits, q, s, N, K), x_dev, y))
        hosts.append((bits, N, q, s))
        ys.append(y)
    st = q4.layer_stack_create(entries, M, q4.Q4_STACK_INDEPENDENT)
    q4.layer_stack_run(st)
    q4.layer_stack_check(st)
    torch.cuda.synchronize()
    for (bits, N, q, s), y in zip(hosts, ys):
        yy = y.cpu().numpy().reshape(M, N)
        if case == "zeros":
            assert np.all(yy == 0.0)
        H.assert_parity(yy, q, s, x, bits)
    st.close()

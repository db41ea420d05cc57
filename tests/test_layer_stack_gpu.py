"""The captured layer stack: same results as one call per product, oracle parity,
and the full 64-layer decode stream (13.7 GB) checked on sampled rows."""
import numpy as np
import pytest

from bit_weight_gemv_q4_b200 import synth, workloads
from bit_weight_gemv_q4_b200.workloads import Tensor
import gpu_helpers as H

pytestmark = pytest.mark.gpu

MIXED = [
    Tensor("a", 4, 1000, 5120, 201), Tensor("b", 8, 37, 96, 202), Tensor("c", 4, 17, 17408, 203),
    Tensor("d", 8, 4099, 5120, 204), Tensor("e", 4, 64, 4096 + 32, 205), Tensor("f", 4, 7168, 5120, 206),
]


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


@pytest.mark.parametrize("M", [1, 4])
def test_stack_equals_single_calls_and_oracle(q4, M):
    torch = H.torch()
    st = workloads.DeviceStream(MIXED, M)
    assert st.stack.launches() == len(MIXED)
    st.run()
    st.check()
    first = [_y(st, i).copy() for i in range(len(MIXED))]
    # a second replay is bitwise identical
    for y in st.y:
        y.fill_(float("nan"))
    st.run()
    st.check()
    for i in range(len(MIXED)):
        assert np.array_equal(_y(st, i), first[i])
    # each product equals a direct call on the same device buffers
    for i, t in enumerate(MIXED):
        ws = H.workspace(t.bits, t.N, t.K, M)
        y = torch.empty(M * t.N, device="cuda")
        (q4.q4_gemv if t.bits == 4 else q4.q8_gemv)(st.packed[i], t.N, t.K, st.x[t.K], M, y, ws)
        q4.q4_workspace_check(ws)
        assert np.array_equal(y.cpu().numpy().reshape(M, t.N), first[i]), t.name
    # and the oracle, on every row
    for i, t in enumerate(MIXED):
        q, s, x = _host_rows(st, i, 0, t.N)
        H.assert_parity(first[i], q, s, x, t.bits)
    # without programmatic dependent launch the results are the same bits
    st2 = workloads.DeviceStream(MIXED, M, flags=q4.Q4_STACK_NO_PDL)
    st2.run()
    st2.check()
    for i in range(len(MIXED)):
        assert np.array_equal(_y(st2, i), first[i])
    st.close()
    st2.close()


@pytest.mark.parametrize("M", [1, 4])
def test_full_decode_stream_sampled(q4, M):
    """All 257 products of one decode step (64 layers + q8 head, 13.7 GB) in the
    captured stack; sampled rows of several tensors against the oracle."""
    torch = H.torch()
    tensors = workloads.decode_stream(fused=True)
    st = workloads.DeviceStream(tensors, M)
    assert st.stack.launches() == 257
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

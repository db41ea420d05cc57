"""The q4 product without a caller workspace (q4_gemv_noalloc).

Some callers cannot allocate device memory where they run the product: a
plug-in inside a host application that owns the device memory budget, or a
latency-critical loop that must not call cudaMalloc (it can synchronise the
whole device).  q4_gemv_noalloc takes its split-tile scratch from a static
device array of the library instead.  These tests call it through the C ABI on
two calls in a row and check each output element against the fp64 oracle
within the product tolerance, and bitwise against q4_gemv (the same kernel,
split and fix-up order, with a workspace the test allocates); NaN guard words
around y catch a write outside it.  The file sorts last so that a run stopping
at the first failure has run every other test first; it also passes on its own
in a fresh process.
"""
import numpy as np
import pytest

import oracle
import gpu_helpers as H

pytestmark = pytest.mark.gpu

CASES = [(1000, 5120, 1), (4099, 512, 4), (17, 17408, 2), (64, 4096 + 32, 3), (34816, 5120, 1)]
GUARD = 64


@pytest.fixture(scope="module")
def q4(cuda_device):
    import bit_weight_gemv_q4_b200 as lib

    return lib


@pytest.mark.parametrize("N,K,M", CASES)
def test_noalloc_matches_the_oracle_and_the_workspace_entry_point(q4, N, K, M):
    torch = H.torch()
    q, s, x = H.host_inputs(4, N, K, M, tensor_id=300 + N % 97)
    packed = H.to_device_packed(4, q, s, N, K)
    x_dev = H.to_device_x(x)
    y_ws, guards_ok = H.run_gemv(4, packed, N, K, x_dev, M)  # q4_gemv with its own workspace
    assert guards_ok
    y_ref, B = oracle.gemv(4, q, s, x)
    for call in range(2):
        full = torch.full((M * N + 2 * GUARD,), float("nan"), dtype=torch.float32, device="cuda")
        q4.q4_gemv_noalloc(packed, N, K, x_dev, M, full[GUARD: GUARD + M * N])
        torch.cuda.synchronize()
        f = full.cpu().numpy()
        assert np.all(np.isnan(f[:GUARD])) and np.all(np.isnan(f[GUARD + M * N:])), f"call {call}: write outside y"
        got = f[GUARD: GUARD + M * N].reshape(M, N)
        ok, _, _ = oracle.within_tolerance(got.astype(np.float64), y_ref, B)
        assert ok.all(), f"call {call}: {(~ok).sum()} outputs outside the oracle's tolerance"
        assert np.array_equal(got, y_ws), f"call {call}: differs from q4_gemv"


def test_noalloc_rejects_shapes_beyond_the_static_array(q4):
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemv_noalloc(1 << 20, 1 << 30, 64, 1 << 20, 1, 1 << 20)
    assert e.value.code == q4.Q4_ERR_UNSUPPORTED
    assert "static array" in str(e.value)

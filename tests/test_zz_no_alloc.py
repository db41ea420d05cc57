"""The q4 product without a caller workspace (q4_gemv_noalloc).

Some callers cannot allocate device memory where they run the product -- for
example inside an open stream capture, or as a plug-in under a host
application's memory budget.  q4_gemv_noalloc takes its split-tile scratch from
a static device array of the library instead.  These tests call it through the
C ABI and compare it with q4_gemv (which uses a workspace the test allocates),
within the tolerance of the other parity tests, on two calls in a row.  The
file sorts last so that a run stopping at the first failure has run every
other test first; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest

import oracle
import gpu_helpers as H

pytestmark = pytest.mark.gpu

CASES = [(1000, 5120, 1), (4099, 512, 4), (17, 17408, 2), (64, 4096 + 32, 3), (34816, 5120, 1)]


@pytest.fixture(scope="module")
def q4(cuda_device):
    import bit_weight_gemv_q4_b200 as lib

    return lib


@pytest.mark.parametrize("N,K,M", CASES)
def test_noalloc_matches_workspace_entry_point(q4, N, K, M):
    torch = H.torch()
    q, s, x = H.host_inputs(4, N, K, M, tensor_id=300 + N % 97)
    packed = H.to_device_packed(4, q, s, N, K)
    x_dev = H.to_device_x(x)
    y_ref, _ = H.run_gemv(4, packed, N, K, x_dev, M)  # q4_gemv with its own workspace
    _, B = oracle.gemv(4, q, s, x)
    for call in range(2):
        y = torch.full((M * N,), float("nan"), device="cuda")
        q4.q4_gemv_noalloc(packed, N, K, x_dev, M, y)
        torch.cuda.synchronize()
        got = y.cpu().numpy().reshape(M, N)
        ok, err, bound = oracle.within_tolerance(got, y_ref.astype(np.float64), B)
        assert ok.all(), f"call {call}: {(~ok).sum()} outputs differ beyond tolerance"


def test_noalloc_rejects_shapes_beyond_the_static_array(q4):
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemv_noalloc(1 << 20, 1 << 30, 64, 1 << 20, 1, 1 << 20)
    assert e.value.code == q4.Q4_ERR_UNSUPPORTED
    assert "static array" in str(e.value)

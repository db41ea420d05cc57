"""Parity of the sm_100a product kernels with the CPU oracle, through the C-ABI.

Tolerance (the pass criterion of the product): |y - y_ref| <= 1e-3 * B + 1e-6
per element, with y_ref and B = sum_k |w x| from the fp64 oracle.  Integer
decoding is checked bit-exactly.
"""
import numpy as np
import pytest

import oracle
from bit_weight_gemv_q4_b200 import synth, workloads
import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4(cuda_device):
    import bit_weight_gemv_q4_b200 as lib

    return lib


def T():
    return H.torch()


# ---------------------------------------------------------------- bounded wait
def test_bounded_wait_gives_up_and_reports(q4):
    # a barrier that nothing completes: the library's wait returns after ~10 ms
    assert q4.q4_selftest_wait_timeout(10_000_000) == 1


# ------------------------------------------------------------ generator / pack
@pytest.mark.parametrize("bits,K,rows", [(4, 5120, (0, 37)), (4, 17408, (4090, 9)), (8, 5120, (248300, 20)), (8, 96, (3, 5))])
def test_device_generator_matches_host(q4, bits, K, rows):
    t = T()
    row0, n = rows
    tid = 77
    q_host, s_host = synth.tensor(bits, 0, tid, row0 + n, K, row0=row0, nrows=n)
    q_dev = t.empty(q_host.size, dtype=t.uint8, device="cuda")
    s_dev = t.empty(s_host.size, dtype=t.int16, device="cuda")
    synth.weights_device(bits, 0, synth.weight_stream(tid), K, row0, n, q_dev)
    synth.scales_device(0, synth.scale_stream(tid), K, row0, n, s_dev)
    x_host = synth.activations(0, synth.act_stream(5), 3, K)
    x_dev = t.empty(x_host.size, dtype=t.int16, device="cuda")
    synth.activations_device(0, synth.act_stream(5), 3, K, x_dev)
    t.cuda.synchronize()
    assert np.array_equal(q_dev.cpu().numpy().view(q_host.dtype).reshape(q_host.shape), q_host)
    assert np.array_equal(s_dev.cpu().numpy().view(np.uint16).reshape(s_host.shape), s_host)
    assert np.array_equal(x_dev.cpu().numpy().view(np.uint16).reshape(x_host.shape), x_host)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(1, 32), (17, 96), (33, 4096 + 32), (1000, 5120)])
def test_device_pack_matches_host_pack(q4, bits, N, K):
    t = T()
    q, s = synth.tensor(bits, 1, 9, N, K)
    ref = q4.q4_pack_weights(bits, q, s, N, K)
    out = t.zeros(ref.size, dtype=t.uint8, device="cuda")
    q4.q4_pack_weights_device(bits, t.from_numpy(q.view(np.uint8).copy()).cuda(),
                              t.from_numpy(s.view(np.int16).copy()).cuda(), N, K, out)
    t.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(1, 32), (16, 64), (17, 96), (45, 4096 + 32), (300, 5120)])
def test_in_register_decode_is_bit_exact(q4, bits, N, K):
    """The kernels' in-register dequantisation returns the generator's integers."""
    t = T()
    q, s = synth.tensor(bits, 2, 11, N, K)
    packed = H.to_device_packed(bits, q, s, N, K)
    q_out = t.full((N * K,), 99, dtype=t.int8, device="cuda")
    s_out = t.zeros(N * (K // 32), dtype=t.int16, device="cuda")
    q4.q4_unpack_device(bits, packed, N, K, q_out, s_out)
    t.cuda.synchronize()
    if bits == 4:
        nib = np.empty((N, K), dtype=np.int64)
        nib[:, 0::2] = q & 0xF
        nib[:, 1::2] = q >> 4
        ints = np.where(nib >= 8, nib - 16, nib)
    else:
        ints = q.astype(np.int64)
    assert np.array_equal(q_out.cpu().numpy().reshape(N, K).astype(np.int64), ints)
    assert np.array_equal(s_out.cpu().numpy().view(np.uint16).reshape(N, K // 32), s)


# ------------------------------------------------------------------- parity
PARITY = [
    (4, 1, 32, 1), (4, 7, 64, 2), (4, 16, 96, 3), (4, 33, 4096 + 32, 4), (4, 1000, 5120, 1), (4, 4099, 512, 4),
    (4, 17, 17408, 1), (4, 24, 17408, 4), (4, 2000, 256, 2),
    (8, 1, 32, 1), (8, 33, 96, 2), (8, 1000, 4096 + 32, 3), (8, 4099, 5120, 4), (8, 16, 17408, 4), (8, 3, 64, 1),
]


@pytest.mark.parametrize("bits,N,K,M", PARITY)
def test_parity_with_oracle(q4, bits, N, K, M):
    q, s, x = H.host_inputs(bits, N, K, M, seed=0, tensor_id=N + K)
    packed = H.to_device_packed(bits, q, s, N, K)
    y, guards = H.run_gemv(bits, packed, N, K, H.to_device_x(x), M)
    assert guards, "write outside y"
    H.assert_parity(y, q, s, x, bits)


def test_single_q4_4096(q4):
    """One q4 4096 x 4096 product at M = 1, whole output against the oracle."""
    (t,) = workloads.single_q4()
    q, s, x = H.host_inputs(4, t.N, t.K, 1, seed=0, tensor_id=t.tensor_id)
    packed = H.to_device_packed(4, q, s, t.N, t.K)
    y, guards = H.run_gemv(4, packed, t.N, t.K, H.to_device_x(x), 1)
    assert guards
    H.assert_parity(y, q, s, x, 4)


@pytest.mark.parametrize("M", [1, 4])
def test_one_layer(q4, M):
    """The seven projections of one 27B-shaped layer, q4, at M = 1 and M = 4."""
    for t in workloads.layer_q4():
        q, s, x = H.host_inputs(4, t.N, t.K, M, seed=0, tensor_id=t.tensor_id)
        packed = H.to_device_packed(4, q, s, t.N, t.K)
        y, guards = H.run_gemv(4, packed, t.N, t.K, H.to_device_x(x), M)
        assert guards, t.name
        H.assert_parity(y, q, s, x, 4)


def _device_tensor(q4, bits, seed, tid, N, K):
    """Generate and pack a full-size tensor on the device."""
    t = T()
    canon = t.empty(N * (K // 2 if bits == 4 else K), dtype=t.uint8, device="cuda")
    scales = t.empty(N * (K // 32), dtype=t.int16, device="cuda")
    synth.weights_device(bits, seed, synth.weight_stream(tid), K, 0, N, canon)
    synth.scales_device(seed, synth.scale_stream(tid), K, 0, N, scales)
    packed = t.empty(q4.q4_packed_bytes(bits, N, K), dtype=t.uint8, device="cuda")
    q4.q4_pack_weights_device(bits, canon, scales, N, K, packed)
    del canon, scales
    return packed


def sampled_rows(N, count=8, seed=0):
    """First and last tiles, plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(16, N))) | set(range(max(0, N - 16), N)) | set(rng.integers(0, N, count).tolist())
    return sorted(rows)


@pytest.mark.parametrize("head", workloads.draft_heads(), ids=lambda h: h.name)
def test_q8_vocab_heads(q4, head):
    """Draft-head projections K=5120 q8 at M=1, the mapped (65,536 rows) and the
    full vocabulary (248,320 rows): every output within the tolerance of the
    oracle (the weights are generated on the device, the oracle's copy is
    regenerated on the host)."""
    t = T()
    seed = 0
    packed = _device_tensor(q4, 8, seed, head.tensor_id, head.N, head.K)
    x = synth.activations(seed, synth.act_stream(head.tensor_id), 1, head.K)
    y, guards = H.run_gemv(8, packed, head.N, head.K, H.to_device_x(x), 1)
    assert guards
    del packed
    t.cuda.empty_cache()
    q, s = synth.tensor(8, seed, head.tensor_id, head.N, head.K)
    H.assert_parity(y, q, s, x, 8)


# --------------------------------------------------------------- edge cases
@pytest.mark.parametrize("fn", ["q4_gemv", "q8_gemv"])
def test_empty_problems(q4, fn):
    t = T()
    y = t.full((8,), 5.0, device="cuda")
    f = getattr(q4, fn)
    f(None, 0, 64, None, 1, y, None)          # N = 0: nothing happens
    f(None, 8, 64, None, 0, y, None)          # M = 0: nothing happens
    f(None, 4, 0, None, 2, y, None)           # K = 0: the empty sum
    t.cuda.synchronize()
    assert t.all(y == 0).item()


@pytest.mark.parametrize("bits", [4, 8])
def test_one_hot_is_exact(q4, bits):
    """x = e_k: y[n] = s[n][k/32] q[n][k], a single exact product -> bit-exact."""
    t = T()
    N, K = 48, 4096 + 32
    q, s, _ = H.host_inputs(bits, N, K, 1, tensor_id=5)
    packed = H.to_device_packed(bits, q, s, N, K)
    ws = H.workspace(bits, N, K, 1)
    for k in [0, 1, 31, 32, 63, 64, 2047, K - 1]:
        x = np.zeros((1, K), dtype=np.uint16)
        x[0, k] = 0x3F80  # 1.0
        y, _ = H.run_gemv(bits, packed, N, K, H.to_device_x(x), 1, ws)
        y_ref, _ = oracle.gemv(bits, q, s, x)
        assert np.array_equal(y.astype(np.float64), y_ref), k
    _ = t


@pytest.mark.parametrize("bits", [4, 8])
def test_linearity_and_determinism(q4, bits):
    N, K, M = 777, 5120, 3
    q, s, x = H.host_inputs(bits, N, K, M, tensor_id=8)
    packed = H.to_device_packed(bits, q, s, N, K)
    ws = H.workspace(bits, N, K, M)
    y1, _ = H.run_gemv(bits, packed, N, K, H.to_device_x(x), M, ws)
    y2, _ = H.run_gemv(bits, packed, N, K, H.to_device_x(x), M, ws)
    assert np.array_equal(y1, y2), "not bitwise reproducible"
    # doubling x doubles every exact product and every partial sum exactly
    xf = (x.astype(np.uint32) << 16).view(np.float32) * 2
    x2 = (xf.view(np.uint32) >> 16).astype(np.uint16)
    y3, _ = H.run_gemv(bits, packed, N, K, H.to_device_x(x2), M, ws)
    assert np.array_equal(y3, 2 * y1)


@pytest.mark.parametrize("bits", [4, 8])
def test_rows_of_m4_are_independent(q4, bits):
    """Identical activation rows give identical outputs; each row of an M=4
    product matches the M=1 product of that row within the tolerance."""
    N, K = 512, 5120
    q, s, x = H.host_inputs(bits, N, K, 4, tensor_id=12)
    packed = H.to_device_packed(bits, q, s, N, K)
    same = np.repeat(x[:1], 4, axis=0)
    y, _ = H.run_gemv(bits, packed, N, K, H.to_device_x(same), 4)
    assert all(np.array_equal(y[0], y[m]) for m in range(1, 4))
    y4, _ = H.run_gemv(bits, packed, N, K, H.to_device_x(x), 4)
    for m in range(4):
        y1, _ = H.run_gemv(bits, packed, N, K, H.to_device_x(x[m:m + 1]), 1)
        H.assert_parity(y1, q, s, x[m:m + 1], bits)
        H.assert_parity(y4[m:m + 1], q, s, x[m:m + 1], bits)


def test_workspace_is_left_zeroed(q4):
    t = T()
    N, K, M = 1000, 5120, 2
    q, s, x = H.host_inputs(4, N, K, M, tensor_id=13)
    packed = H.to_device_packed(4, q, s, N, K)
    ws = H.workspace(4, N, K, M)
    H.run_gemv(4, packed, N, K, H.to_device_x(x), M, ws)
    # the status word and the tile counters (the workspace's tail) are zero
    # again; partial sums in between may remain
    T_tiles = (N + 15) // 16
    counters = (4 * T_tiles + 255) // 256 * 256
    assert t.all(ws[:4] == 0).item()
    assert t.all(ws[ws.numel() - counters:] == 0).item()
    # a larger shape reuses the same workspace prefix: its counters start zero
    q2, s2, x2 = H.host_inputs(8, 4099, 5120, 1, tensor_id=15)
    p2 = H.to_device_packed(8, q2, s2, 4099, 5120)
    ws2 = H.workspace(8, 4099, 5120, 1)
    for (bits, pk, n, k, xx, m, qq, ss) in [(4, packed, N, K, x, M, q, s), (8, p2, 4099, 5120, x2, 1, q2, s2)] * 2:
        y, _ = H.run_gemv(bits, pk, n, k, H.to_device_x(xx), m, ws2)
        H.assert_parity(y, qq, ss, xx, bits)


def test_bad_workspace_is_rejected(q4):
    t = T()
    N, K = 64, 64
    q, s, x = H.host_inputs(4, N, K, 1, tensor_id=14)
    packed = H.to_device_packed(4, q, s, N, K)
    y = t.empty(N, device="cuda")
    small = t.zeros(16, dtype=t.uint8, device="cuda")
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemv(packed, N, K, H.to_device_x(x), 1, y, small)
    assert e.value.code == q4.Q4_ERR_BUFFER_TOO_SMALL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [1, 4])
def test_degenerate_rows(q4, bits, M):
    N, K = 96, 5120
    q, s = H.degenerate_rows(bits, N, K)
    x = synth.activations(3, synth.act_stream(41), M, K)
    y, ok = H.run_gemv(bits, H.to_device_packed(bits, q, s, N, K), N, K, H.to_device_x(x), M)
    assert ok
    H.assert_parity(y, q, s, x, bits)

"""Offline repack: bit-exact against the layout specification, exact inverse."""
import numpy as np
import pytest

import bit_weight_gemv_q4_b200 as q4
from bit_weight_gemv_q4_b200 import synth, workloads
from oracle import layout

SHAPES = [(1, 32), (7, 64), (16, 96), (17, 160), (33, 32), (100, 256), (48, 4096 + 32)]


def canonical_ints(bits, q, K):
    if bits == 8:
        return q.astype(np.int64)
    lo = (q & 0xF).astype(np.int64)
    hi = (q >> 4).astype(np.int64)
    out = np.empty((q.shape[0], K), dtype=np.int64)
    out[:, 0::2], out[:, 1::2] = lo, hi
    return np.where(out >= 8, out - 16, out)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", SHAPES)
def test_pack_matches_layout_spec_and_round_trips(bits, N, K):
    q, s = synth.tensor(bits, 3, 40 + N, N, K)
    packed = q4.q4_pack_weights(bits, q, s, N, K)
    assert packed.size == q4.q4_packed_bytes(bits, N, K)
    qd, sd = layout.decode(bits, packed, N, K)
    assert np.array_equal(qd, canonical_ints(bits, q, K))
    assert np.array_equal(sd, s)
    assert layout.padding_is_zero(bits, packed, N, K)
    q2, s2 = q4.q4_unpack_weights(bits, packed, N, K)
    assert np.array_equal(q2, q) and np.array_equal(s2, s)


@pytest.mark.parametrize("bits", [4, 8])
def test_every_code_at_every_position(bits):
    """Each integer value in every slot, word and nibble/byte position."""
    N, K = 32, 64
    lo, hi = (-8, 7) if bits == 4 else (-128, 127)
    vals = np.arange(lo, hi + 1)
    s = np.full((N, K // 32), 0x3C00, dtype=np.uint16)
    for shift in range(len(vals)):
        ints = vals[(np.arange(N * K) + shift) % len(vals)].reshape(N, K)
        if bits == 4:
            nib = (ints & 0xF).astype(np.uint8)
            qc = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
        else:
            qc = ints.astype(np.int8)
        packed = q4.q4_pack_weights(bits, qc, s, N, K)
        qd, _ = layout.decode(bits, packed, N, K)
        assert np.array_equal(qd, ints)


def test_sizes_equal_algorithmic_bytes_without_padding():
    for t in workloads.decode_stream(fused=True) + workloads.layer_q4() + workloads.single_q4() + workloads.draft_heads():
        assert q4.q4_packed_bytes(t.bits, t.N, t.K) == t.bytes, t
    # padding only adds whole tiles / chunks
    assert q4.q4_packed_bytes(4, 17, 96) == 1 * 2 * 1152
    assert q4.q4_packed_bytes(8, 33, 96) == 2 * 3 * 1088


def test_invalid_arguments():
    assert q4.q4_packed_bytes(5, 16, 32) == 0  # 5 bits need K % 64 == 0
    assert q4.q4_packed_bytes(7, 16, 64) == 0
    assert q4.q4_packed_bytes(4, 16, 48) == 0
    assert q4.q4_packed_bytes(4, -1, 32) == 0
    q, s = synth.tensor(4, 0, 1, 16, 64)
    lib = q4.lib()
    out = np.zeros(100, dtype=np.uint8)
    assert lib.q4_pack_weights(4, q.ctypes.data, s.ctypes.data, 16, 64, out.ctypes.data, out.size) == q4.Q4_ERR_BUFFER_TOO_SMALL
    assert lib.q4_pack_weights(7, q.ctypes.data, s.ctypes.data, 16, 64, out.ctypes.data, out.size) == q4.Q4_ERR_INVALID_ARG
    assert lib.q4_pack_weights(4, q.ctypes.data, s.ctypes.data, 16, 40, out.ctypes.data, out.size) == q4.Q4_ERR_SHAPE
    assert lib.q4_pack_weights(4, None, s.ctypes.data, 16, 64, out.ctypes.data, out.size) == q4.Q4_ERR_INVALID_ARG
    assert "null" in q4.q4_last_error()
    # empty tensors are valid and produce nothing
    assert q4.q4_packed_bytes(4, 0, 64) == 0 and q4.q4_packed_bytes(4, 16, 0) == 0
    assert lib.q4_pack_weights(4, None, None, 0, 64, None, 0) == q4.Q4_OK

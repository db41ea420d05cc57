"""Python binding of the seeded synthetic-input generator (``csrc/synth.cu``).

Every array returned is in the canonical (interchange) layout:

* q4 weights: ``uint8 [N][K/2]``, element k in byte k/2, low nibble for even k,
  4-bit two's complement (values -8..7);
* q8 weights: ``int8 [N][K]``;
* group scales: ``uint16 [N][K/32]`` holding fp16 bits;
* activations: ``uint16 [M][K]`` holding bf16 bits.

Streams identify tensors: one (seed, stream) pair per weight tensor, a separate
stream for its scales and one per activation block, so any row of any tensor
can be regenerated on its own.  The ``*_device`` functions write the same bits
into device memory (torch CUDA tensors), for workloads too large to generate on
the host.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None

SCALE_STD = 0.02


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build_synth()
        L = ctypes.CDLL(path)
        i64, u64 = ctypes.c_int64, ctypes.c_uint64
        vp = ctypes.c_void_p
        L.synth_q4.argtypes = [u64, u64, i64, i64, i64, vp]
        L.synth_q8.argtypes = [u64, u64, i64, i64, i64, vp]
        L.synth_scales.argtypes = [u64, u64, i64, i64, i64, ctypes.c_double, vp]
        L.synth_bf16_normals.argtypes = [u64, u64, i64, i64, vp]
        L.synth_normals_f64.argtypes = [u64, u64, i64, i64, vp]
        L.synth_f64_to_f16_array.argtypes = [vp, i64, vp]
        L.synth_f64_to_bf16_array.argtypes = [vp, i64, vp]
        L.synth_words.argtypes = [u64, u64, i64, i64, vp]
        L.synth_log_array.argtypes = [vp, i64, vp]
        L.synth_cos2pi_array.argtypes = [vp, i64, vp]
        L.synth_q4_device.argtypes = [u64, u64, i64, i64, i64, vp, vp]
        L.synth_q8_device.argtypes = [u64, u64, i64, i64, i64, vp, vp]
        L.synth_scales_device.argtypes = [u64, u64, i64, i64, i64, ctypes.c_double, vp, vp]
        L.synth_bf16_normals_device.argtypes = [u64, u64, i64, i64, vp, vp]
        L.synth_e4m3_scales.argtypes = [u64, u64, i64, i64, i64, vp]
        L.synth_e4m3_scales_device.argtypes = [u64, u64, i64, i64, i64, vp, vp]
        for f in (L.synth_q4, L.synth_q8, L.synth_scales, L.synth_bf16_normals, L.synth_normals_f64,
                  L.synth_q4_device, L.synth_q8_device, L.synth_scales_device, L.synth_bf16_normals_device):
            f.restype = ctypes.c_int
        for f in (L.synth_f64_to_f16_array, L.synth_f64_to_bf16_array, L.synth_words, L.synth_log_array,
                  L.synth_cos2pi_array):
            f.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def weights(bits: int, seed: int, stream: int, K: int, row0: int, nrows: int) -> np.ndarray:
    """Canonical quantised weights for rows [row0, row0+nrows) of a tensor with K columns.
    q5 / q6 (int8 [nrows][K] in [-16, 15] / [-32, 31]): the q8 codes of the
    same stream shifted right by 3 / 2 (arithmetic)."""
    if bits in (5, 6):
        return weights(8, seed, stream, K, row0, nrows) >> np.int8(8 - bits)
    if bits == 4:
        out = np.empty((nrows, K // 2), dtype=np.uint8)
        rc = lib().synth_q4(seed, stream, K, row0, nrows, _ptr(out))
    elif bits == 8:
        out = np.empty((nrows, K), dtype=np.int8)
        rc = lib().synth_q8(seed, stream, K, row0, nrows, _ptr(out))
    else:
        raise ValueError("bits must be 4 or 8")
    if rc != 0:
        raise ValueError(f"synth: bad shape K={K} row0={row0} nrows={nrows}")
    return out


def scales(seed: int, stream: int, K: int, row0: int, nrows: int, std: float = SCALE_STD) -> np.ndarray:
    """fp16 bits of the group scales |std * N(0,1)|, shape [nrows][K/32]."""
    out = np.empty((nrows, K // 32), dtype=np.uint16)
    if lib().synth_scales(seed, stream, K, row0, nrows, float(std), _ptr(out)) != 0:
        raise ValueError(f"synth: bad shape K={K}")
    return out


def activations(seed: int, stream: int, M: int, K: int) -> np.ndarray:
    """bf16 bits of M activation rows of N(0,1), shape [M][K]."""
    out = np.empty((M, K), dtype=np.uint16)
    if lib().synth_bf16_normals(seed, stream, 0, M * K, _ptr(out)) != 0:
        raise ValueError("synth: bad activation shape")
    return out


def normals_f64(seed: int, stream: int, i0: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.float64)
    lib().synth_normals_f64(seed, stream, i0, count, _ptr(out))
    return out


def words(seed: int, stream: int, i0: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.uint64)
    lib().synth_words(seed, stream, i0, count, _ptr(out))
    return out


def log_f64(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty_like(a)
    lib().synth_log_array(_ptr(a), a.size, _ptr(out))
    return out


def cos2pi_f64(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty_like(a)
    lib().synth_cos2pi_array(_ptr(a), a.size, _ptr(out))
    return out


def f64_to_f16_bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().synth_f64_to_f16_array(_ptr(a), a.size, _ptr(out))
    return out


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().synth_f64_to_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


# ----------------------------------------------------------------------------
# Stream identifiers of the workloads.  Each weight tensor has one id t; its
# quantised values use stream 2t and its scales stream 2t+1.  Activations use
# streams from ACT_STREAM_BASE up.
# ----------------------------------------------------------------------------
ACT_STREAM_BASE = 1 << 20


def weight_stream(tensor_id: int) -> int:
    return 2 * tensor_id


def scale_stream(tensor_id: int) -> int:
    return 2 * tensor_id + 1


def act_stream(k_id: int) -> int:
    return ACT_STREAM_BASE + k_id


def e4m3_scales(seed: int, stream: int, K: int, row0: int, nrows: int) -> np.ndarray:
    """E4M3 bytes of NVFP4 block scales (0.25 .. 3.75), shape [nrows][K/16]."""
    out = np.empty((nrows, K // 16), dtype=np.uint8)
    if lib().synth_e4m3_scales(seed, stream, K, row0, nrows, _ptr(out)) != 0:
        raise ValueError(f"synth: bad shape K={K}")
    return out


# the per-tensor scale of every synthetic NVFP4 tensor (fp32): with codes of
# magnitude up to 6 and block scales up to 3.75, weights stay below 0.23
NVFP4_TENSOR_SCALE = 0.01


def nvfp4_tensor(seed: int, tensor_id: int, N: int, K: int, row0: int = 0, nrows: int | None = None):
    """(canonical codes [nrows][K/2], E4M3 block scales [nrows][K/16], tensor scale) of a synthetic NVFP4 tensor:
    uniform codes (every 4-bit pattern) from the q4 code stream of the tensor id, scales from its scale stream."""
    if nrows is None:
        nrows = N - row0
    c = weights(4, seed, weight_stream(tensor_id), K, row0, nrows)
    s = e4m3_scales(seed, scale_stream(tensor_id), K, row0, nrows)
    return c, s, NVFP4_TENSOR_SCALE


def tensor(bits: int, seed: int, tensor_id: int, N: int, K: int, row0: int = 0, nrows: int | None = None):
    """(canonical q, fp16 scale bits) of one synthetic weight tensor (or a row slice of it)."""
    if nrows is None:
        nrows = N - row0
    q = weights(bits, seed, weight_stream(tensor_id), K, row0, nrows)
    s = scales(seed, scale_stream(tensor_id), K, row0, nrows)
    return q, s


# ----------------------------------------------------------------------------
# device-side generation (same bits, written into torch CUDA tensors)
# ----------------------------------------------------------------------------
def _dev(t) -> int:
    if not getattr(t, "is_cuda", False) or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


class _null_ctx:
    def __enter__(self):
        return None

    def __exit__(self, *a):
        return False


def _dev_check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"synth {what}: {'bad arguments' if rc == -1 else 'CUDA launch failed'}")


def weights_device(bits: int, seed: int, stream_id: int, K: int, row0: int, nrows: int, out, stream=None) -> None:
    """Canonical weights of rows [row0, row0+nrows) into `out` (uint8 [nrows][K/2] or int8 [nrows][K])."""
    expect = nrows * (K // 2 if bits == 4 else K)
    if out.numel() * out.element_size() < expect:
        raise ValueError("output tensor too small")
    fn = lib().synth_q4_device if bits == 4 else lib().synth_q8_device
    _dev_check(fn(seed, stream_id, K, row0, nrows, _dev(out), _stream(stream)), "weights")
    if bits in (5, 6):  # the q8 codes shifted right (arithmetic), as weights() does on the host
        import torch

        with torch.cuda.stream(stream) if stream is not None else _null_ctx():
            v = out.view(torch.int8)[:expect]
            v.copy_(torch.bitwise_right_shift(v, 8 - bits))


def scales_device(seed: int, stream_id: int, K: int, row0: int, nrows: int, out, std: float = SCALE_STD,
                  stream=None) -> None:
    if out.numel() * out.element_size() < 2 * nrows * (K // 32):
        raise ValueError("output tensor too small")
    _dev_check(lib().synth_scales_device(seed, stream_id, K, row0, nrows, float(std), _dev(out), _stream(stream)),
               "scales")


def e4m3_scales_device(seed: int, stream_id: int, K: int, row0: int, nrows: int, out, stream=None) -> None:
    if out.numel() * out.element_size() < nrows * (K // 16):
        raise ValueError("output tensor too small")
    _dev_check(lib().synth_e4m3_scales_device(seed, stream_id, K, row0, nrows, _dev(out), _stream(stream)), "e4m3 scales")


def activations_device(seed: int, stream_id: int, M: int, K: int, out, stream=None) -> None:
    if out.numel() * out.element_size() < 2 * M * K:
        raise ValueError("output tensor too small")
    _dev_check(lib().synth_bf16_normals_device(seed, stream_id, 0, M * K, _dev(out), _stream(stream)), "activations")


__all__ = [
    "weights_device", "scales_device", "activations_device", "log_f64", "cos2pi_f64",
    "weights", "scales", "activations", "normals_f64", "words", "f64_to_f16_bits", "f64_to_bf16_bits",
    "tensor", "weight_stream", "scale_stream", "act_stream", "SCALE_STD", "lib",
    "e4m3_scales", "e4m3_scales_device", "nvfp4_tensor", "NVFP4_TENSOR_SCALE",
]

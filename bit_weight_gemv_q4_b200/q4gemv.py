"""Python binding of the q4gemv C-ABI library (``libq4gemv.so``).

Argument marshalling only: every step of the product runs in the library's
CUDA kernels, and the functions here carry the C names.  Device buffers are
torch CUDA tensors (or raw integer device addresses); host buffers are numpy
arrays.  There is no CPU fallback: if the library cannot be loaded, importing
this package raises, and GPU calls without a usable sm_100 device raise
:class:`Q4Error`.

See ``include/q4gemv.h`` for the operation, the layouts and the error codes.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

Q4_OK = 0
Q4_ERR_INVALID_ARG = -1
Q4_ERR_SHAPE = -2
Q4_ERR_ALIGN = -3
Q4_ERR_BUFFER_TOO_SMALL = -4
Q4_ERR_CUDA = -5
Q4_ERR_TIMEOUT = -6
Q4_ERR_UNSUPPORTED = -7
Q4_STACK_NO_PDL = 1
Q4_STACK_GRAPH = 2
Q4_STACK_INDEPENDENT = 4
Q4_STACK_ORDERED = 32
Q4_CHAIN_PERSISTENT = 8
Q4_CHAIN_GRAPH = 16
Q4_QUANT_ABSMAX = 0
Q4_QUANT_SIGNED_MAX = 1
Q4_OP_PRODUCT = 0
Q4_OP_RESIDUAL_RMSNORM = 1
Q4_OP_SWIGLU = 2
Q4_FMT_NVFP4 = 16
Q4_SPEC_MAX_DRAFT = 15

ERROR_NAMES = {
    Q4_ERR_INVALID_ARG: "INVALID_ARG",
    Q4_ERR_SHAPE: "SHAPE",
    Q4_ERR_ALIGN: "ALIGN",
    Q4_ERR_BUFFER_TOO_SMALL: "BUFFER_TOO_SMALL",
    Q4_ERR_CUDA: "CUDA",
    Q4_ERR_TIMEOUT: "TIMEOUT",
    Q4_ERR_UNSUPPORTED: "UNSUPPORTED",
}

# Symbols include/q4gemv.h declares (checked by the tests against the header).
EXPORTED = [
    "q4_last_error", "q4_packed_bytes", "q4_pack_weights", "q4_pack_weights_device", "q4_unpack_weights",
    "q4_gemv_workspace_bytes",
    "q4_gemv", "q8_gemv", "q4_gemv_noalloc", "q4_workspace_check", "q4_set_wait_timeout_ns", "q4_unpack_device",
    "q4_selftest_wait_timeout", "layer_stack_create", "layer_stack_run", "layer_stack_check",
    "layer_stack_launches", "layer_stack_destroy", "q4_quantize", "q4_quantize_device", "layer_chain_create",
    "q4_residual_rmsnorm", "q4_swiglu", "q4_nvfp4_packed_bytes", "q4_pack_nvfp4", "q4_unpack_nvfp4",
    "q4_pack_nvfp4_device", "q4_nvfp4_dequant_device", "q4_gather_rows_device", "q4_spec_draft", "q4_spec_verify",
]


class Q4Error(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{ERROR_NAMES.get(code, code)}: {message}")
        self.code = code


class StackEntry(ctypes.Structure):
    _fields_ = [
        ("bits", ctypes.c_int),
        ("N", ctypes.c_int64),
        ("K", ctypes.c_int64),
        ("packed", ctypes.c_void_p),
        ("x", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
    ]


class ChainOp(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int),
        ("bits", ctypes.c_int),
        ("N", ctypes.c_int64),
        ("K", ctypes.c_int64),
        ("packed", ctypes.c_void_p),
        ("inp", ctypes.c_void_p),
        ("out", ctypes.c_void_p),
        ("resid", ctypes.c_void_p),
    ]


def _load() -> ctypes.CDLL:
    path = _build.GEMV_LIB
    if not os.path.exists(path) or _build._stale(path, _build.GEMV_DEPS):
        try:
            _build.build_gemv()
        except Exception as exc:  # no silent fallback: the product needs its CUDA library
            raise ImportError(f"libq4gemv.so is missing and could not be built: {exc}") from exc
    L = ctypes.CDLL(path)
    i32, i64, u64, sz, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p
    sig = {
        "q4_last_error": ([], ctypes.c_char_p),
        "q4_packed_bytes": ([i32, i64, i64], sz),
        "q4_pack_weights": ([i32, vp, vp, i64, i64, vp, sz], i32),
        "q4_pack_weights_device": ([i32, vp, vp, i64, i64, vp, sz, vp], i32),
        "q4_unpack_weights": ([i32, vp, sz, i64, i64, vp, vp], i32),
        "q4_gemv_workspace_bytes": ([i32, i64, i64, i32], sz),
        "q4_gemv": ([vp, i64, i64, vp, i32, vp, vp, sz, vp], i32),
        "q8_gemv": ([vp, i64, i64, vp, i32, vp, vp, sz, vp], i32),
        "q4_gemv_noalloc": ([vp, i64, i64, vp, i32, vp, vp], i32),
        "q4_workspace_check": ([vp, sz, vp], i32),
        "q4_set_wait_timeout_ns": ([u64], i32),
        "q4_unpack_device": ([i32, vp, i64, i64, vp, vp, vp], i32),
        "q4_selftest_wait_timeout": ([u64, ctypes.POINTER(i32)], i32),
        "layer_stack_create": ([ctypes.POINTER(StackEntry), i32, i32, i32, ctypes.POINTER(vp)], i32),
        "layer_stack_run": ([vp, vp], i32),
        "layer_stack_check": ([vp, vp], i32),
        "layer_stack_launches": ([vp], i32),
        "layer_stack_destroy": ([vp], None),
        "q4_quantize": ([i32, i32, vp, i64, i64, vp, vp], i32),
        "layer_chain_create": ([ctypes.POINTER(ChainOp), i32, i32, i32, ctypes.POINTER(vp)], i32),
        "q4_residual_rmsnorm": ([vp, vp, vp, vp, i64, i32, i32, vp], i32),
        "q4_swiglu": ([vp, vp, i64, i32, vp], i32),
        "q4_quantize_device": ([i32, i32, vp, i64, i64, vp, vp, vp], i32),
        "q4_nvfp4_packed_bytes": ([i64, i64], sz),
        "q4_pack_nvfp4": ([vp, vp, ctypes.c_float, i64, i64, vp, sz], i32),
        "q4_unpack_nvfp4": ([vp, sz, i64, i64, vp, vp, ctypes.POINTER(ctypes.c_float)], i32),
        "q4_pack_nvfp4_device": ([vp, vp, ctypes.c_float, i64, i64, vp, sz, vp], i32),
        "q4_nvfp4_dequant_device": ([vp, i64, i64, vp, vp], i32),
        "q4_gather_rows_device": ([vp, i64, i64, vp, i64, vp, vp], i32),
        "q4_spec_draft": ([vp, i64, vp, ctypes.c_float, vp, vp, vp, vp, vp], i32),
        "q4_spec_verify": ([vp, i64, vp, i64, vp, vp, vp, i32, ctypes.c_float, vp, vp, vp], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def q4_last_error() -> str:
    return _lib.q4_last_error().decode()


def _check(rc: int) -> None:
    if rc != Q4_OK:
        raise Q4Error(rc, q4_last_error())


def _dev_ptr(t) -> int:
    """Device address of a torch CUDA tensor (or an int address, or None -> 0)."""
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    if not getattr(t, "is_cuda", False):
        raise Q4Error(Q4_ERR_INVALID_ARG, "expected a CUDA tensor")
    return t.data_ptr()


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _stream(stream) -> int:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------------------
# host-side packing
# ----------------------------------------------------------------------------
def q4_packed_bytes(bits: int, N: int, K: int) -> int:
    return int(_lib.q4_packed_bytes(bits, N, K))


def q4_pack_weights(bits: int, canon_q: np.ndarray, scales_fp16: np.ndarray, N: int, K: int) -> np.ndarray:
    """Canonical q and fp16 scale bits (numpy, host) -> packed bytes (numpy uint8)."""
    q = np.ascontiguousarray(canon_q, dtype=np.uint8 if bits == 4 else np.int8)
    s = np.ascontiguousarray(scales_fp16, dtype=np.uint16)
    expect_q = (N, K // 2) if bits == 4 else (N, K)
    if q.size != expect_q[0] * expect_q[1] or s.size != N * (K // 32):
        raise Q4Error(Q4_ERR_SHAPE, f"canonical arrays do not match N={N} K={K}")
    out = np.zeros(max(q4_packed_bytes(bits, N, K), 1), dtype=np.uint8)
    _check(_lib.q4_pack_weights(bits, q.ctypes.data, s.ctypes.data, N, K, out.ctypes.data, out.size))
    return out[: q4_packed_bytes(bits, N, K)]


def q4_pack_weights_device(bits: int, canon_q, scales_fp16, N: int, K: int, out, stream=None) -> None:
    """Canonical q and fp16 scale bits (device tensors) -> packed bytes in `out` (device)."""
    _check(_lib.q4_pack_weights_device(bits, _dev_ptr(canon_q), _dev_ptr(scales_fp16), N, K, _dev_ptr(out),
                                       _nbytes(out), _stream(stream)))


def q4_unpack_weights(bits: int, packed: np.ndarray, N: int, K: int) -> tuple[np.ndarray, np.ndarray]:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    q = np.zeros((N, K // 2) if bits == 4 else (N, K), dtype=np.uint8 if bits == 4 else np.int8)
    s = np.zeros((N, K // 32), dtype=np.uint16)
    _check(_lib.q4_unpack_weights(bits, packed.ctypes.data, packed.size, N, K, q.ctypes.data, s.ctypes.data))
    return q, s


def q4_nvfp4_packed_bytes(N: int, K: int) -> int:
    return int(_lib.q4_nvfp4_packed_bytes(N, K))


def q4_pack_nvfp4(codes: np.ndarray, scales: np.ndarray, tensor_scale: float, N: int, K: int) -> np.ndarray:
    """NVFP4 canonical codes [N][K/2], E4M3 scale bytes [N][K/16] and the fp32
    tensor scale (host) -> packed bytes (numpy uint8)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    sc = np.ascontiguousarray(scales, dtype=np.uint8)
    if c.size != N * (K // 2) or sc.size != N * (K // 16):
        raise Q4Error(Q4_ERR_SHAPE, f"canonical NVFP4 arrays do not match N={N} K={K}")
    n = q4_nvfp4_packed_bytes(N, K)
    out = np.zeros(max(n, 1), dtype=np.uint8)
    _check(_lib.q4_pack_nvfp4(c.ctypes.data, sc.ctypes.data, float(tensor_scale), N, K, out.ctypes.data, out.size))
    return out[:n]


def q4_unpack_nvfp4(packed: np.ndarray, N: int, K: int) -> tuple[np.ndarray, np.ndarray, float]:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    c = np.zeros((N, K // 2), dtype=np.uint8)
    sc = np.zeros((N, K // 16), dtype=np.uint8)
    t = ctypes.c_float(0.0)
    _check(_lib.q4_unpack_nvfp4(packed.ctypes.data, packed.size, N, K, c.ctypes.data, sc.ctypes.data,
                                ctypes.byref(t)))
    return c, sc, t.value


def q4_pack_nvfp4_device(codes, scales, tensor_scale: float, N: int, K: int, out, stream=None) -> None:
    """The NVFP4 repack on device tensors."""
    _check(_lib.q4_pack_nvfp4_device(_dev_ptr(codes), _dev_ptr(scales), float(tensor_scale), N, K, _dev_ptr(out),
                                     _nbytes(out), _stream(stream)))


def q4_nvfp4_dequant_device(packed, N: int, K: int, w_out, stream=None) -> None:
    """Debug decoder: the fp32 weights [N][K] the product kernels multiply."""
    _check(_lib.q4_nvfp4_dequant_device(_dev_ptr(packed), N, K, _dev_ptr(w_out), _stream(stream)))


def q4_gather_rows_device(src, row_bytes: int, n_src: int, rows, n_rows: int, dst, stream=None) -> None:
    """dst row r = src row rows[r] (row_bytes bytes each), device tensors."""
    _check(_lib.q4_gather_rows_device(_dev_ptr(src), row_bytes, n_src, _dev_ptr(rows), n_rows, _dev_ptr(dst),
                                      _stream(stream)))


def q4_spec_draft(z, n_map: int, vmap, temperature: float, u, row_out, token_out, q_out, stream=None) -> None:
    """One draft token from the draft head's mapped logits z (device tensors)."""
    _check(_lib.q4_spec_draft(_dev_ptr(z), n_map, _dev_ptr(vmap), float(temperature), _dev_ptr(u),
                              _dev_ptr(row_out), _dev_ptr(token_out), _dev_ptr(q_out), _stream(stream)))


def q4_spec_verify(target, V: int, drafts, n_map: int, vmap, inv_map, rows, n_draft: int, temperature: float, u,
                   out, stream=None) -> None:
    """Keep / reject n_draft drafted tokens against the main model's logits;
    out (int32, 3 n_draft + 3) receives the kept count, the emitted tokens and
    the per-position decisions (see include/q4gemv.h)."""
    opt = lambda t: 0 if t is None else _dev_ptr(t)  # noqa: E731
    _check(_lib.q4_spec_verify(_dev_ptr(target), V, opt(drafts), n_map, opt(vmap), opt(inv_map), opt(rows), n_draft,
                               float(temperature), _dev_ptr(u), _dev_ptr(out), _stream(stream)))


def q4_quantize(bits: int, mode: int, w_bf16: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16 weight bits [N][K] (numpy, host) -> (canonical codes, fp16 scale bits [N][K/32])."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    q = np.zeros((N, K // 2) if bits == 4 else (N, K), dtype=np.uint8 if bits == 4 else np.int8)
    s = np.zeros((N, max(K // 32, 0)), dtype=np.uint16)
    _check(_lib.q4_quantize(bits, mode, w.ctypes.data, N, K, q.ctypes.data, s.ctypes.data))
    return q, s


def q4_quantize_device(bits: int, mode: int, w_bf16, N: int, K: int, canon_q_out, scales_out, stream=None) -> None:
    """The same on device tensors (bf16 bits [N][K] in, canonical codes and scales out)."""
    _check(_lib.q4_quantize_device(bits, mode, _dev_ptr(w_bf16), N, K, _dev_ptr(canon_q_out), _dev_ptr(scales_out),
                                   _stream(stream)))


# ----------------------------------------------------------------------------
# device-side product
# ----------------------------------------------------------------------------
def q4_gemv_workspace_bytes(bits: int, N: int, K: int, M: int) -> int:
    n = int(_lib.q4_gemv_workspace_bytes(bits, N, K, M))
    if n == 0:
        raise Q4Error(Q4_ERR_INVALID_ARG, q4_last_error())
    return n


def _gemv(fn, packed, N, K, x, M, y, workspace, stream):
    _check(fn(_dev_ptr(packed), N, K, _dev_ptr(x), M, _dev_ptr(y), _dev_ptr(workspace),
              _nbytes(workspace) if workspace is not None and not isinstance(workspace, int) else 0,
              _stream(stream)))


def q4_gemv(packed, N: int, K: int, x, M: int, y, workspace, stream=None) -> None:
    """y[M][N] (fp32, device) = W x for packed q4 W and bf16 x [M][K] (device)."""
    _gemv(_lib.q4_gemv, packed, N, K, x, M, y, workspace, stream)


def q8_gemv(packed, N: int, K: int, x, M: int, y, workspace, stream=None) -> None:
    """y[M][N] (fp32, device) = W x for packed q8 W and bf16 x [M][K] (device)."""
    _gemv(_lib.q8_gemv, packed, N, K, x, M, y, workspace, stream)


def q4_gemv_noalloc(packed, N: int, K: int, x, M: int, y, stream=None) -> None:
    """q4_gemv with the library's static scratch array instead of a workspace
    (for callers that cannot allocate device memory where they run)."""
    _check(_lib.q4_gemv_noalloc(_dev_ptr(packed), N, K, _dev_ptr(x), M, _dev_ptr(y), _stream(stream)))


def q4_workspace_check(workspace, stream=None) -> None:
    _check(_lib.q4_workspace_check(_dev_ptr(workspace), _nbytes(workspace), _stream(stream)))


def q4_set_wait_timeout_ns(ns: int) -> None:
    _check(_lib.q4_set_wait_timeout_ns(int(ns)))


def q4_unpack_device(bits: int, packed, N: int, K: int, q_out, scales_out, stream=None) -> None:
    _check(_lib.q4_unpack_device(bits, _dev_ptr(packed), N, K, _dev_ptr(q_out), _dev_ptr(scales_out),
                                 _stream(stream)))


def q4_selftest_wait_timeout(timeout_ns: int) -> int:
    out = ctypes.c_int(-1)
    _check(_lib.q4_selftest_wait_timeout(int(timeout_ns), ctypes.byref(out)))
    return out.value


# ----------------------------------------------------------------------------
# layer stack
# ----------------------------------------------------------------------------
class LayerStack:
    """Owner of a captured q4_stack; keeps the entry tensors alive."""

    def __init__(self, handle: int, keepalive):
        self.handle = handle
        self._keepalive = keepalive

    def launches(self) -> int:
        return int(_lib.layer_stack_launches(self.handle))

    def close(self) -> None:
        if self.handle:
            _lib.layer_stack_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def layer_stack_create(entries, M: int, flags: int = 0) -> LayerStack:
    """entries: sequence of (bits, N, K, packed, x, y) with device tensors."""
    arr = (StackEntry * max(len(entries), 1))()
    keep = []
    for i, (bits, N, K, packed, x, y) in enumerate(entries):
        arr[i] = StackEntry(bits, N, K, _dev_ptr(packed), _dev_ptr(x), _dev_ptr(y))
        keep.append((packed, x, y))
    h = ctypes.c_void_p(0)
    _check(_lib.layer_stack_create(arr, len(entries), M, flags, ctypes.byref(h)))
    return LayerStack(h.value, keep)


def layer_chain_create(ops, M: int, flags: int = 0) -> LayerStack:
    """ops: sequence of (kind, bits, N, K, packed, inp, out, resid); device
    tensors, raw addresses or None (NULL)."""
    arr = (ChainOp * max(len(ops), 1))()
    keep = []
    for i, (kind, bits, N, K, packed, inp, out, resid) in enumerate(ops):
        ptr = lambda t: 0 if t is None else _dev_ptr(t)  # noqa: E731
        arr[i] = ChainOp(kind, bits, N, K, ptr(packed), ptr(inp), ptr(out), ptr(resid))
        keep.append((packed, inp, out, resid))
    h = ctypes.c_void_p(0)
    _check(_lib.layer_chain_create(arr, len(ops), M, flags, ctypes.byref(h)))
    return LayerStack(h.value, keep)


def q4_residual_rmsnorm(h, y, gamma, x, N: int, M: int, set_: bool = False, stream=None) -> None:
    """h (fp32 [M][N]) <- h + y (or y when set_); x (bf16 bits [M][N]) = RMSNorm(h) * gamma."""
    _check(_lib.q4_residual_rmsnorm(_dev_ptr(h), _dev_ptr(y), _dev_ptr(gamma), _dev_ptr(x), N, M, int(set_),
                                    _stream(stream)))


def q4_swiglu(y_gu, x, N: int, M: int, stream=None) -> None:
    """x (bf16 bits [M][N]) = silu(gate) * up from y_gu (fp32 [M][2N])."""
    _check(_lib.q4_swiglu(_dev_ptr(y_gu), _dev_ptr(x), N, M, _stream(stream)))


def layer_stack_run(stack: LayerStack, stream=None) -> None:
    _check(_lib.layer_stack_run(stack.handle, _stream(stream)))


def layer_stack_check(stack: LayerStack, stream=None) -> None:
    _check(_lib.layer_stack_check(stack.handle, _stream(stream)))


def layer_stack_destroy(stack: LayerStack) -> None:
    stack.close()


__all__ = [
    "Q4Error", "LayerStack", "StackEntry", "EXPORTED", "lib", "q4_last_error", "q4_packed_bytes",
    "q4_pack_weights", "q4_pack_weights_device", "q4_unpack_weights", "q4_gemv_workspace_bytes", "q4_gemv", "q8_gemv",
    "q4_gemv_noalloc",
    "q4_workspace_check", "q4_set_wait_timeout_ns", "q4_unpack_device", "q4_selftest_wait_timeout",
    "layer_stack_create", "layer_stack_run", "layer_stack_check", "layer_stack_destroy",
    "q4_quantize", "q4_quantize_device", "Q4_QUANT_ABSMAX", "Q4_QUANT_SIGNED_MAX",
    "layer_chain_create", "Q4_CHAIN_PERSISTENT", "Q4_CHAIN_GRAPH", "ChainOp", "Q4_OP_PRODUCT", "Q4_OP_RESIDUAL_RMSNORM", "Q4_OP_SWIGLU",
    "q4_residual_rmsnorm", "q4_swiglu", "Q4_FMT_NVFP4", "q4_nvfp4_packed_bytes", "q4_pack_nvfp4", "q4_unpack_nvfp4",
    "q4_pack_nvfp4_device", "q4_nvfp4_dequant_device", "Q4_SPEC_MAX_DRAFT", "q4_gather_rows_device",
    "q4_spec_draft", "q4_spec_verify",
]

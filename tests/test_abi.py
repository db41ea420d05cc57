"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching a device (no GPU needed)."""
import os
import re
import subprocess

import numpy as np
import pytest

import bit_weight_gemv_q4_b200 as q4
from bit_weight_gemv_q4_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "q4gemv.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"Q4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_declarations_match_binding():
    assert declared_symbols() == sorted(q4.EXPORTED)


def test_every_declared_symbol_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", build.GEMV_LIB], stdout=subprocess.PIPE, text=True, check=True)
    exported = {line.split()[-1] for line in out.stdout.splitlines() if line.strip()}
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(q4.lib(), name)


def test_only_declared_symbols_are_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", build.GEMV_LIB], stdout=subprocess.PIPE, text=True, check=True)
    ours = {line.split()[-1] for line in out.stdout.splitlines() if " T " in line}
    assert {s for s in ours if s.startswith(("q4_", "q8_", "layer_stack_", "layer_chain_"))} == set(declared_symbols())


# Host-side validation happens before any CUDA call, so these run without a GPU.
ALIGNED = 1 << 20  # a fake, 16-byte-aligned device address (never dereferenced)


@pytest.mark.parametrize("fn", ["q4_gemv", "q8_gemv"])
def test_argument_errors_are_detected_on_the_host(fn):
    f = getattr(q4.lib(), fn)
    ws = 1 << 20
    # M outside 0..4
    assert f(ALIGNED, 16, 64, ALIGNED, 5, ALIGNED, ALIGNED, ws, None) == q4.Q4_ERR_INVALID_ARG
    assert f(ALIGNED, 16, 64, ALIGNED, -1, ALIGNED, ALIGNED, ws, None) == q4.Q4_ERR_INVALID_ARG
    # K not a multiple of 32, negative sizes
    assert f(ALIGNED, 16, 48, ALIGNED, 1, ALIGNED, ALIGNED, ws, None) == q4.Q4_ERR_SHAPE
    assert f(ALIGNED, -16, 64, ALIGNED, 1, ALIGNED, ALIGNED, ws, None) == q4.Q4_ERR_SHAPE
    # null pointers
    assert f(None, 16, 64, ALIGNED, 1, ALIGNED, ALIGNED, ws, None) == q4.Q4_ERR_INVALID_ARG
    assert f(ALIGNED, 16, 64, None, 1, ALIGNED, ALIGNED, ws, None) == q4.Q4_ERR_INVALID_ARG
    assert f(ALIGNED, 16, 64, ALIGNED, 1, None, ALIGNED, ws, None) == q4.Q4_ERR_INVALID_ARG
    assert f(ALIGNED, 16, 64, ALIGNED, 1, ALIGNED, None, ws, None) == q4.Q4_ERR_INVALID_ARG
    # misaligned operands
    assert f(ALIGNED + 8, 16, 64, ALIGNED, 1, ALIGNED, ALIGNED, ws, None) == q4.Q4_ERR_ALIGN
    assert f(ALIGNED, 16, 64, ALIGNED + 2, 1, ALIGNED, ALIGNED, ws, None) == q4.Q4_ERR_ALIGN
    assert f(ALIGNED, 16, 64, ALIGNED, 1, ALIGNED + 2, ALIGNED, ws, None) == q4.Q4_ERR_ALIGN
    assert f(ALIGNED, 16, 64, ALIGNED, 1, ALIGNED, ALIGNED + 4, ws, None) == q4.Q4_ERR_ALIGN
    assert q4.q4_last_error()
    # empty problems are no-ops and touch nothing
    assert f(None, 0, 64, None, 1, None, None, 0, None) == q4.Q4_OK
    assert f(None, 16, 64, None, 0, None, None, 0, None) == q4.Q4_OK


def test_stack_argument_errors():
    lib = q4.lib()
    import ctypes

    h = ctypes.c_void_p(0)
    assert lib.layer_stack_create(None, 1, 1, 0, ctypes.byref(h)) == q4.Q4_ERR_INVALID_ARG
    arr = (q4.StackEntry * 1)()
    assert lib.layer_stack_create(arr, 1, 0, 0, ctypes.byref(h)) == q4.Q4_ERR_INVALID_ARG
    assert lib.layer_stack_create(arr, 1, 5, 0, ctypes.byref(h)) == q4.Q4_ERR_INVALID_ARG
    assert lib.layer_stack_run(None, None) == q4.Q4_ERR_INVALID_ARG
    lib.layer_stack_destroy(None)


def test_without_a_device_gpu_calls_fail_loudly():
    """No silent CPU fallback: on a host without a usable device the product
    entry points return an error (there is nothing else they could do)."""
    try:
        import torch

        if torch.cuda.is_available():
            pytest.skip("a device is present")
    except ImportError:
        pass
    rc = q4.lib().q4_gemv(ALIGNED, 16, 64, ALIGNED, 1, ALIGNED, ALIGNED, 1 << 20, None)
    assert rc in (q4.Q4_ERR_CUDA, q4.Q4_ERR_UNSUPPORTED)
    with pytest.raises(q4.Q4Error):
        q4.q4_gemv_workspace_bytes(4, 16, 64, 1)
    _ = np  # numpy imported for parity with other test modules


def test_binding_structs_match_the_c_layout(tmp_path):
    """The ctypes structures the binding passes by pointer (q4_stack_entry,
    q4_chain_op) have the sizes and field offsets the C compiler gives the
    header's declarations (compiled here as C99 with gcc)."""
    import ctypes
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc is not available")
    cases = [
        ("q4_stack_entry", q4.StackEntry, {"bits": "bits", "N": "N", "K": "K", "packed": "packed", "x": "x", "y": "y"}),
        ("q4_chain_op", q4.ChainOp, {"kind": "kind", "bits": "bits", "N": "N", "K": "K", "packed": "packed",
                                     "inp": "in", "out": "out", "resid": "resid"}),
    ]
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "q4gemv.h"', "int main(void) {"]
    for cname, _, fields in cases:
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for cfield in fields.values():
            lines.append(f'  printf("{cname} {cfield} %zu\\n", offsetof({cname}, {cfield}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        name, field, value = line.split()
        got[(name, field)] = int(value)
    for cname, cls, fields in cases:
        assert ctypes.sizeof(cls) == got[(cname, "size")], cname
        for pyfield, cfield in fields.items():
            assert getattr(cls, pyfield).offset == got[(cname, cfield)], (cname, cfield)


def _c_category(decl: str) -> str:
    decl = " ".join(decl.split())
    if "*" in decl:
        return "ptr"
    words = [w for w in decl.split() if w != "const"]
    if len(words) > 1 and words[-1] not in ("int", "long", "float", "double", "void"):
        words = words[:-1]  # drop the parameter name
    t = " ".join(words)
    return {"int": "int", "int64_t": "i64", "uint64_t": "u64", "size_t": "u64", "unsigned long long": "u64",
            "float": "float", "void": "void"}[t]


def _ctypes_category(t) -> str:
    import ctypes

    if t is None:
        return "void"
    if t in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(t, "_type_") and isinstance(t._type_, type):
        return "ptr"
    return {ctypes.c_int: "int", ctypes.c_int64: "i64", ctypes.c_uint64: "u64", ctypes.c_size_t: "u64",
            ctypes.c_float: "float"}[t]


def test_binding_signatures_match_the_c_prototypes():
    """Every declared entry point is called through ctypes with the argument
    and return types of its C prototype (int, int64_t, 64-bit unsigned,
    float, pointer), in order."""
    text = re.sub(r"/\*.*?\*/", " ", open(HEADER).read(), flags=re.S)
    protos = re.findall(r"Q4_API\s+([\w\s\*]+?)\b(\w+)\s*\(([^)]*)\)\s*;", text)
    assert sorted(name for _, name, _ in protos) == declared_symbols()
    L = q4.lib()
    for ret, name, params in protos:
        params = params.strip()
        c_args = [] if params in ("", "void") else [_c_category(p) for p in params.split(",")]
        f = getattr(L, name)
        assert [_ctypes_category(a) for a in f.argtypes] == c_args, name
        assert _ctypes_category(f.restype) == _c_category(ret), name

"""bit_weight_gemv_q4_b200 -- group-quantised weight x activation products for
single-user decode on NVIDIA B200 (sm_100a).

* :mod:`.q4gemv`    -- Python binding of the C-ABI library ``libq4gemv.so``
  (``q4_pack_weights``, ``q4_gemv``, ``q8_gemv``, ``layer_stack_run`` ...);
  the names below resolve to it lazily.
* :mod:`.synth`     -- seeded synthetic inputs in the canonical layout.
* :mod:`.workloads` -- the tensor shapes of the decode workloads.
* :mod:`.build`     -- in-tree build of the native libraries.
"""
from __future__ import annotations

import importlib


_SUBMODULES = ("build", "q4gemv", "synth", "workloads")


def __getattr__(name):
    if name.startswith("_"):
        raise AttributeError(name)
    if name in _SUBMODULES:  # `from package import build` must not load the library first
        return importlib.import_module(f".{name}", __name__)
    mod = importlib.import_module(".q4gemv", __name__)
    try:
        return getattr(mod, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None

"""B200-native (sm_100a) WKV kernels for RWKV time mixing.

The CUDA library ``libwkv_b200.so`` (built from ``csrc/``) exposes a small C
ABI declared in ``include/wkv.h``; ``rwkv_wkv_linear_mix_b200.wkv`` is the thin
ctypes binding over it. ``synth`` draws the seeded synthetic inputs.
Submodules are imported lazily so that ``synth`` can be used without the
CUDA library.
"""

import importlib

__all__ = ["wkv", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    if name in ("wkv4_forward", "wkv4_backward", "wkv4_chunk_step", "wkv4_state_init",
                "wkv6_forward"):
        return getattr(importlib.import_module(f"{__name__}.wkv"), name)
    raise AttributeError(name)

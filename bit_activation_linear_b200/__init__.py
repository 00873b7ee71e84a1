"""BitLinear / H-BitLinear forward (BitNet b1.58, BitNet v2) for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libbitnet_b200.so`` built from ``csrc/``; the
Python functions in :mod:`.binding` only marshal torch tensors into its entry points.  The
library is loaded on first use, so ``import bit_activation_linear_b200.synth`` works on a
machine without a GPU.
"""
from . import synth  # noqa: F401

__all__ = ["synth"]


def __getattr__(name):
    if name.startswith("bitnet_") or name in ("BitnetError", "load_library"):
        import importlib
        return getattr(importlib.import_module(".binding", __name__), name)
    raise AttributeError(name)

"""B200-native token-skipping denoising step for masked diffusion LMs.

The compute path is libdllm.so (hand-written sm_100a CUDA behind a C ABI,
include/dllm.h); this package only marshals torch tensors into it.
"""
from ._lib import load, DllmError, make_config  # noqa: F401

__all__ = ["load", "DllmError", "make_config", "Engine", "ops"]


def __getattr__(name):
    if name == "Engine":
        from .engine import Engine
        return Engine
    if name == "ops":
        from . import ops
        return ops
    raise AttributeError(name)

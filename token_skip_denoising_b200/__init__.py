"""B200-native token-skipping denoising step for masked diffusion LMs.

The compute path is libdllm.so (hand-written sm_100a CUDA behind a C ABI,
include/dllm.h); this package only marshals torch tensors into it.
Submodules: `engine` (the generation engine), `ops` (single kernels).
"""
from ._lib import load, DllmError, make_config  # noqa: F401

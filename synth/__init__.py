"""Seeded synthetic workloads shared by the oracle and the CUDA path.

This package holds shapes and random draws only: no step of the denoising
method is computed here.  Both `oracle/` and `token_skip_denoising_b200/`
read their inputs from it, and neither imports the other.
"""
from .configs import ModelDims, RunConfig, CONFIGS, get_config  # noqa: F401
from .gen import (  # noqa: F401
    make_weights, make_prompt, make_tokens, microbench_hidden,
    microbench_active, lock_pattern, WEIGHT_SEED, PROMPT_SEED,
)

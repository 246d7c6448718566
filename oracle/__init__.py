"""CPU oracle for the token-skipping denoising step (test infrastructure only).

This package is the plain, slow, fp64 statement of what the CUDA path
computes.  Only the tests, the smoke check of `__graft_entry__` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` may import it; the
library itself never does, and the oracle imports nothing from the library.
Inputs come from the seeded generators in `synth/`.

Sources followed (page title, section):
  * "ES-dLLM: Efficient Inference for Diffusion Large Language Models by
    Early-Skipping" (gist.science summary), sec. 2.1, Eq. 1 and the partial
    cache update / early skip, sec. 2.2 periodic refresh.
  * "SureLock: Stopping Computation for Converged Tokens" summary, sec. 2.1
    lock condition, skip, attention over locked K/V.
  * dLLM-Cache explainer (aibr.jp), sec. 3 core technique: long-interval
    prompt cache, similarity-gated partial response update, ratio rho.
  * "Plan for Speed: Dilated Scheduling for Masked Diffusion Language Models"
    summary, sec. 2 algorithm design (R = ceil(log_a B) rounds of
    non-adjacent positions) and the hallway example in the lay summary.

Parity pins: every function is pinned by a `-m "not gpu"` test in
tests/test_oracle_*.py against closed forms, brute force, the pages' worked
example or invariants.  The transformer backbone (RMSNorm, RoPE, SwiGLU,
untied LM head) is not on the pages; its shapes come from the workload
descriptions and its formulas are the textbook ones, pinned by closed forms.
"""

"""Failure detection and checkpoint / resume, in forms that fault, trap or hang no GPU.

* A grid-wide phase wait of the fused layer kernel is made unsatisfiable (its
  counter is set far below zero, a flag nothing will raise) with a short poll
  limit: the kernel records DLLM_DEV_TIMEOUT, every CTA stops its work, waits
  for its own copies in flight, frees its tensor memory and returns; the host
  reads the status, and the next launch, with the default limit, computes the
  same layers as an engine that never timed out.
* The whole generation state is the caller-owned state buffer, the token
  buffer and the schedule position: copying them into a fresh handle resumes
  the generation bit for bit (kernel-per-step layer, whose sums are
  deterministic).
"""
import numpy as np
import pytest
import torch

from synth import get_config, make_tokens, make_weights

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from token_skip_denoising_b200._lib import DllmError
    from token_skip_denoising_b200.engine import Engine, device_status

DEV = "cuda"
TINY = get_config("tiny")
DEV_TIMEOUT = 1


def _rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


@pytest.mark.parametrize("name", ["tiny", "llada3"])
def test_fused_phase_wait_runs_out_and_the_next_launch_is_clean(name):
    from synth.configs import scaled
    cfg = TINY if name == "tiny" else scaled(get_config("llada_es"), n_layers=3, vocab=2048,
                                             mask_id=2047).replace(skip_layer=2)
    w = make_weights(cfg.model, device=DEV)
    tok0 = make_tokens(cfg).to(DEV)
    eng = Engine(cfg, w, tok0.clone().contiguous(), layer_kernel="fused")
    ref = Engine(cfg, w, tok0.clone().contiguous(), layer_kernel="fused")
    ls = cfg.skip_layer
    for e in (eng, ref):
        e.step()                                        # refresh (kernel-per-step path: all rows)
        assert e.begin_step() == "skip"
    torch.cuda.synchronize()
    assert device_status() == 0
    h0 = eng.buffer("hidden").clone()
    kc0, vc0 = eng.buffer("kcache").clone(), eng.buffer("vcache").clone()
    sync = eng.buffer("fused_sync")
    assert int(sync.abs().sum()) == 0                   # counters are zero between launches
    eng.set_wait_limit(20000)                           # a few ms instead of ~0.4 s
    sync[0] = -(1 << 30)                                # the first phase of the launch can never complete
    eng.layers_forward(0, ls)                           # one fused launch over layers 0 .. ls-1
    torch.cuda.synchronize()
    assert device_status() == DEV_TIMEOUT
    assert device_status() == 0                         # read and cleared
    assert int(sync.abs().sum()) == 0                   # the last CTA out cleared every counter
    # nothing was written: the rows' hidden state and every cache row are as before
    assert torch.equal(eng.buffer("hidden"), h0)
    assert torch.equal(eng.buffer("kcache"), kc0) and torch.equal(eng.buffer("vcache"), vc0)
    # the next launch with the default limit runs the same layers as an engine that never timed out
    eng.set_wait_limit(0)
    eng.layers_forward(0, ls)
    ref.layers_forward(0, ls)
    torch.cuda.synchronize()
    assert device_status() == 0
    n = int(eng.buffer("nrows")[0])
    rows = eng.buffer("rows")[:n].long()
    assert _rel(eng.buffer("hidden")[rows], ref.buffer("hidden")[rows]) < 1e-2   # fp32 sums land in any order
    for c in ("kcache", "vcache"):
        assert _rel(eng.buffer(c)[:ls], ref.buffer(c)[:ls]) < 1e-2
    # and the rest of the generation proceeds normally
    eng.select_layers_forward()
    eng.unmask()
    while not eng.done:
        eng.step()
    torch.cuda.synchronize()
    assert device_status() == 0
    assert not bool((eng.tokens == cfg.model.mask_id).any())


@pytest.mark.parametrize("policy", ["es", "surelock", "dllm_cache"])
def test_checkpoint_resume_is_bit_exact(policy):
    over = {"es": {}, "surelock": {"kl_eps": 1e30, "conf_tau": -1.0},
            "dllm_cache": {"prompt_interval": 3, "sim_tau": 0.99, "rho_cap": 0.5}}[policy]
    cfg = TINY.replace(policy=policy, block_len=8, tokens_per_step=2, **over)
    w = make_weights(cfg.model, device=DEV)
    tok0 = make_tokens(cfg).to(DEV)
    A = Engine(cfg, w, tok0.clone().contiguous(), layer_kernel="split")
    for _ in range(6):
        A.step()
    torch.cuda.synchronize()
    ck_state, ck_tok, ck_prog = A.state.clone(), A.tokens.clone(), A.progress()
    assert ck_prog == {"step": 6, "block": 1, "step_in_block": 2}
    A.generate()
    B = Engine(cfg, w, tok0.clone().contiguous(), layer_kernel="split")
    B.state.copy_(ck_state)
    B.tokens.copy_(ck_tok)
    B.set_progress(ck_prog)
    B.generate()
    torch.cuda.synchronize()
    assert A.progress() == B.progress()
    assert torch.equal(A.tokens, B.tokens)
    for buf in ("kcache", "vcache", "conf", "argmax"):
        assert torch.equal(A.buffer(buf), B.buffer(buf)), buf
    if policy == "surelock":
        assert torch.equal(A.buffer("lock"), B.buffer("lock")) and int(A.buffer("lock").sum()) > 0
    assert not bool((B.tokens == cfg.model.mask_id).any())


def test_progress_outside_the_schedule_is_refused():
    cfg = TINY.replace(block_len=8, tokens_per_step=2)
    eng = Engine(cfg, make_weights(cfg.model, device=DEV), make_tokens(cfg).to(DEV).contiguous())
    for bad in ({"step": 0, "block": 5, "step_in_block": 0}, {"step": 0, "block": 0, "step_in_block": 4},
                {"step": -1, "block": 0, "step_in_block": 0}, {"step": 0, "block": 4, "step_in_block": 1}):
        with pytest.raises(DllmError):
            eng.set_progress(bad)
    eng.begin_step()
    with pytest.raises(DllmError):                     # not in the middle of a step
        eng.set_progress({"step": 0, "block": 0, "step_in_block": 0})
    eng.layers_forward(0, cfg.model.n_layers)
    eng.unmask()
    eng.set_progress({"step": 0, "block": 4, "step_in_block": 0})   # the end of the schedule
    assert eng.done

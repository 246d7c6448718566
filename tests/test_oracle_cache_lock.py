"""Pins of the oracle parts that the step-level invariants cannot see.

* the dLLM-Cache value probe reads the V rows of the fused QKV weight, not the
  K rows (dLLM-Cache explainer sec. 3: features of the response rows);
* a dLLM-Cache partial step with a binding threshold and cap keeps the cached
  K/V and layer outputs of the rows it does not select, and runs the layer on
  the selected rows' carried inputs (dLLM-Cache explainer sec. 3);
* the vocabulary projection computed in chunks equals the one-shot product
  for a vocabulary that is not a multiple of the chunk;
* the SureLock lock rule fires exactly when a row is lock-eligible and has a
  previous distribution (SureLock summary sec. 2.1 item 2, with the threshold
  and the confidence bound made always true).
"""
import math

import numpy as np
import pytest
import torch

from oracle.model import OracleModel, rmsnorm
from oracle.steps import OracleRun
from synth import get_config, make_tokens, make_weights
from synth.configs import ModelDims

TINY = get_config("tiny")


def _toy_dims():
    # 2 heads of dim 2, d = 4: q rows 0-3, k rows 4-7, v rows 8-11 of w_qkv
    return ModelDims(n_layers=1, d_model=4, n_heads=2, n_kv_heads=2, head_dim=2,
                     ffn_dim=4, vocab=8, mask_id=7, rms_eps=0.0)


def _toy_weights(g_attn):
    w_qkv = torch.tensor([[10.0 * r + c for c in range(4)] for r in range(12)])
    return {"w_qkv": w_qkv[None], "w_o": torch.zeros(1, 4, 4), "w_gu": torch.zeros(1, 8, 4),
            "w_down": torch.zeros(1, 4, 4), "g_attn": torch.tensor([g_attn]),
            "g_ffn": torch.ones(1, 4), "g_final": torch.ones(4), "layers": [0]}


def test_value_probe_reads_the_v_rows():
    """v = W_v RMSNorm(h): with h = (2, 2, 2, 2) and eps = 0 the norm is (1, 1, 1, 1), so v_j is
    the sum of row 8 + j of w_qkv, i.e. 40 (8 + j) + 6; with the gain (1, 0, 0, 0) only column 0
    survives, i.e. 10 (8 + j).  K rows would give 166.. / 40.., q rows 6.. / 0.."""
    model = OracleModel(_toy_dims(), _toy_weights([1.0, 1.0, 1.0, 1.0]))
    v = model.value_only(0, np.array([[2.0, 2.0, 2.0, 2.0]]))
    np.testing.assert_array_equal(v, [[326.0, 366.0, 406.0, 446.0]])
    model = OracleModel(_toy_dims(), _toy_weights([1.0, 0.0, 0.0, 0.0]))
    v = model.value_only(0, np.array([[2.0, 2.0, 2.0, 2.0], [-3.0, -3.0, -3.0, -3.0]]))
    np.testing.assert_array_equal(v, [[80.0, 90.0, 100.0, 110.0], [-80.0, -90.0, -100.0, -110.0]])


def test_chunked_vocabulary_projection_matches_one_product():
    """A vocabulary of 40000 rows in chunks of 16384 (two full chunks and a ragged tail) gives
    the same logits as one product of the whole matrix, column for column."""
    d, V = 32, 40000
    dims = ModelDims(n_layers=1, d_model=d, n_heads=2, n_kv_heads=2, head_dim=16,
                     ffn_dim=64, vocab=V, mask_id=V - 1)
    g = torch.Generator().manual_seed(7)
    lm = (0.02 * torch.randn(V, d, generator=g)).to(torch.bfloat16)
    gf = 1.0 + 0.1 * torch.randn(d, generator=g)
    model = OracleModel(dims, {"lm_head": lm, "g_final": gf, "layers": []})
    h = np.random.default_rng(3).standard_normal((3, d))
    z = model.logits(h, chunk=16384)
    zn = h / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + dims.rms_eps) * gf.double().numpy()
    want = zn @ lm.double().numpy().T
    assert z.shape == (3, V)
    np.testing.assert_allclose(z, want, rtol=1e-12, atol=1e-15)
    # the columns on both sides of each chunk edge and the last one
    for c in (0, 16383, 16384, 32767, 32768, V - 1):
        np.testing.assert_allclose(z[:, c], zn @ lm[c].double().numpy(), rtol=1e-12, atol=1e-15)


def _partial_step_case():
    cfg = TINY.replace(policy="dllm_cache", sim_tau=0.5, rho_cap=0.25, prompt_interval=1000,
                       tokens_per_step=4)
    w = make_weights(cfg.model, gain_jitter=0.1)
    tok = make_tokens(cfg).numpy()
    return cfg, w, tok


def test_dllm_cache_partial_step_keeps_unselected_rows():
    """Forced similarities: 12 of the 32 response rows score below tau = 0.5 and the cap is
    ceil(0.25 * 32) = 8, so the 8 lowest of those 12 are recomputed at each layer.  Every other
    row keeps its K/V and its cached output of that layer bit for bit; a selected row's output
    is the layer applied to its carried input (the current output of the previous layer, or its
    embedding at layer 0), and the layer writes the selected rows' K/V before attention."""
    cfg, w, tok = _partial_step_case()
    m = cfg.model
    run = OracleRun(cfg, w, tok)
    run.step()                                            # step 0: full refresh of every row
    run.step()                                            # a partial step, to move the caches on
    K0, V0, H0 = run.K.copy(), run.V.copy(), run.h_cache.copy()
    tok0 = run.tokens.copy()
    n, s = cfg.gen_len, cfg.prompt_len
    rng = np.random.default_rng(11)
    forced, want_sel = [], []
    for l in range(m.n_layers):
        sims = np.full(n, 0.9)
        low = rng.choice(n, 12, replace=False)
        vals = rng.permutation(np.linspace(0.05, 0.45, 12))
        sims[low] = vals
        forced.append(sims)
        want_sel.append(np.sort(low[np.argsort(vals)[:8]]))
    rec = run.step(forced_scores=forced)
    assert rec["kind"] == "partial"
    model = OracleModel(m, w)
    pos_all = np.arange(s, cfg.seq_len)
    x = model.embed(tok0[0, s:])
    for l in range(m.n_layers):
        sel = rec["layers"][l]["sel"]
        np.testing.assert_array_equal(sel, want_sel[l])
        unsel = np.setdiff1d(np.arange(n), sel)
        Kc, Vc = K0[l].copy(), V0[l].copy()
        out = model.layer(l, x[sel], np.zeros(len(sel), np.int64), pos_all[sel], Kc, Vc)
        # the whole cache equals the pre-step cache with only the selected rows rewritten
        np.testing.assert_array_equal(run.K[l], Kc)
        np.testing.assert_array_equal(run.V[l], Vc)
        np.testing.assert_array_equal(run.K[l][0, :, pos_all[unsel]], K0[l][0, :, pos_all[unsel]])
        np.testing.assert_array_equal(run.h_cache[l][0, pos_all[unsel]], H0[l][0, pos_all[unsel]])
        np.testing.assert_array_equal(run.h_cache[l][0, pos_all[sel]], out)
        np.testing.assert_array_equal(run.h_cache[l][0, :s], H0[l][0, :s])     # prompt rows untouched
        x = run.h_cache[l][0, pos_all].copy()


def test_surelock_rule_locks_on_the_first_eligible_step_with_a_previous_distribution():
    """kl_eps = 1e30 and conf_tau = -1 make "KL < eps and conf > tau" true wherever a KL exists.
    A row is lock-eligible once unmasked at the start of a step and has a KL once a distribution
    of it was stored in an earlier step.  So nothing locks at step 0 (no previous distribution);
    at step 1 the prompt and the positions committed at step 0 lock; at every later step t exactly
    the positions committed at step t - 1 lock (their masked-row distribution of step t - 1 is the
    previous one).  A locked row is then never recomputed."""
    cfg = TINY.replace(policy="surelock", kl_eps=1e30, conf_tau=-1.0, tokens_per_step=4)
    w = make_weights(cfg.model)
    tok = make_tokens(cfg).numpy()
    run = OracleRun(cfg, w, tok)
    prev_lock = np.zeros_like(run.lock)
    committed_prev = []
    t = 0
    while not run.done:
        rec = run.step()
        new = set(map(tuple, np.argwhere(run.lock & ~prev_lock).tolist()))
        if t == 0:
            want = set()
        elif t == 1:
            want = {(0, p) for p in range(cfg.prompt_len)} | {(b, p) for b, p, _ in committed_prev}
        else:
            want = {(b, p) for b, p, _ in committed_prev}
        assert new == want, t
        assert set(map(tuple, np.array(rec["new_lock"]).reshape(-1, 2).tolist())) == want
        # the rows computed this step were exactly the rows unlocked at its start
        rows = set(zip(rec["rows"][0].tolist(), rec["rows"][1].tolist()))
        assert rows == set(map(tuple, np.argwhere(~prev_lock).tolist()))
        committed_prev = rec["committed"]
        prev_lock = run.lock.copy()
        t += 1
    assert t == cfg.gen_len // cfg.tokens_per_step
    # every prompt row and every position committed before the last step ends locked
    assert run.lock[0, :cfg.prompt_len].all()
    assert int(run.lock.sum()) == cfg.seq_len - cfg.tokens_per_step

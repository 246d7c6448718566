"""Step-level pins of the oracle: the invariants the method fixes.

* a skipping step that keeps every row reproduces the full-recompute step
  exactly (ES keep = 1, SureLock eps = 0, dLLM-Cache rho = 1 with tau = inf);
* each masked position is unmasked exactly once, in gen_len / n steps
  (DUS: (G / B) * R);
* locked rows never change;
* a skip step rewrites only the rows it recomputes.
"""
import numpy as np
import pytest
import torch

from oracle.steps import OracleRun, generate
from synth import get_config, make_tokens, make_weights
from synth.configs import scaled

TINY = get_config("tiny")


@pytest.fixture(scope="module")
def tiny_w():
    return make_weights(TINY.model)


@pytest.fixture(scope="module")
def tiny_tok():
    return make_tokens(TINY).numpy()


@pytest.fixture(scope="module")
def vanilla(tiny_w, tiny_tok):
    return generate(TINY.replace(policy="vanilla"), tiny_w, tiny_tok)


def _same_run(a, b):
    np.testing.assert_array_equal(a.tokens, b.tokens)
    np.testing.assert_array_equal(a.K, b.K)
    np.testing.assert_array_equal(a.V, b.V)
    assert a.unmask_events == b.unmask_events


def test_es_keep_all_equals_vanilla(tiny_w, tiny_tok, vanilla):
    es = generate(TINY.replace(keep_ratio=1.0, cand_scope="all"), tiny_w, tiny_tok)
    _same_run(es, vanilla)
    np.testing.assert_array_equal(es.conf, vanilla.conf)


def test_surelock_eps_zero_equals_vanilla(tiny_w, tiny_tok, vanilla):
    sl = generate(TINY.replace(policy="surelock", kl_eps=0.0, conf_tau=-1.0), tiny_w, tiny_tok)
    _same_run(sl, vanilla)
    assert not sl.lock.any()


def test_dllm_cache_full_ratio_equals_vanilla(tiny_w, tiny_tok, vanilla):
    cfg = TINY.replace(policy="dllm_cache", sim_tau=float("inf"), rho_cap=1.0,
                       prompt_interval=1000, cand_scope="all")
    dc = generate(cfg, tiny_w, tiny_tok)
    _same_run(dc, vanilla)


@pytest.mark.parametrize("policy", ["vanilla", "es", "surelock", "dllm_cache"])
def test_each_masked_position_unmasked_once(tiny_w, tiny_tok, policy):
    cfg = TINY.replace(policy=policy)
    run = generate(cfg, tiny_w, tiny_tok)
    pos = sorted((b, p) for _, b, p, _ in run.unmask_events)
    assert pos == [(0, p) for p in range(cfg.prompt_len, cfg.seq_len)]
    assert run.n_steps == cfg.gen_len // cfg.tokens_per_step
    assert not np.any(run.tokens == cfg.model.mask_id)
    np.testing.assert_array_equal(run.tokens[:, :cfg.prompt_len], tiny_tok[:, :cfg.prompt_len])
    for _, b, p, t in run.unmask_events:
        assert run.tokens[b, p] == t and t != cfg.model.mask_id


def test_dus_generation_step_count(tiny_w):
    cfg = TINY.replace(block_len=8, unmask="dus", policy="dllm_cache", prompt_interval=5)
    tok = make_tokens(cfg).numpy()
    run = generate(cfg, tiny_w, tok)
    assert run.n_steps == (cfg.gen_len // 8) * 3
    pos = sorted(p for _, _, p, _ in run.unmask_events)
    assert pos == list(range(cfg.prompt_len, cfg.seq_len))
    # within a block, round r commits exactly the positions of the r-th dilated group
    first = [p - cfg.prompt_len for s, _, p, _ in run.unmask_events if s < 3]
    assert sorted(first) == [0, 1, 2, 3, 4, 5, 6, 7]
    r0 = sorted(p - cfg.prompt_len for s, _, p, _ in run.unmask_events if s == 0)
    assert r0 == [0, 4]


def test_locked_rows_never_change(tiny_w, tiny_tok):
    cfg = TINY.replace(policy="surelock", tokens_per_step=2)
    pattern = np.zeros((1, cfg.seq_len), bool)
    pattern[0, ::3] = True                         # a seeded third of the positions lock when eligible
    run = OracleRun(cfg, tiny_w, tiny_tok, lock_pattern=pattern)
    snap = {}
    n_locked = 0
    while not run.done:
        run.step()
        for b, p in zip(*np.nonzero(run.lock)):
            key = (int(b), int(p))
            if key not in snap:
                snap[key] = (run.tokens[b, p], run.K[:, b, :, p].copy(), run.V[:, b, :, p].copy(),
                             run.prev_logits[key][0].copy())
            tok, K, V, z = snap[key]
            assert run.tokens[b, p] == tok
            np.testing.assert_array_equal(run.K[:, b, :, p], K)
            np.testing.assert_array_equal(run.V[:, b, :, p], V)
            np.testing.assert_array_equal(run.prev_logits[key][0], z)
        n_locked = max(n_locked, int(run.lock.sum()))
    assert n_locked > 5
    # locked rows are excluded from the recomputed row set
    assert len(run.last["rows"][1]) == cfg.seq_len - int(run.lock.sum()) or run.done


def test_surelock_all_positions_lock_scope(tiny_w, tiny_tok):
    """Lock scope 'all positions' (the SureLock summary's "each token position i", kept as a flag):
    masked positions lock too.  A locked masked position is never recomputed, its K/V and stored
    distribution never change, and it is still unmasked, exactly once, with the argmax stored when
    it locked; with eps = 0 nothing locks (KL >= 0 and the rule is strict)."""
    cfg = TINY.replace(policy="surelock", tokens_per_step=2, lock_masked=True)
    pattern = np.zeros((1, cfg.seq_len), bool)
    pattern[0, 1::3] = True
    run = OracleRun(cfg, tiny_w, tiny_tok, lock_pattern=pattern)
    snap, locked_masked = {}, {}
    while not run.done:
        masked_before = run.tokens == cfg.model.mask_id
        run.step()
        for b, p in zip(*np.nonzero(run.lock)):
            key = (int(b), int(p))
            if key not in snap:
                snap[key] = (run.K[:, b, :, p].copy(), run.V[:, b, :, p].copy(), run.prev_logits[key][0].copy())
                if masked_before[b, p]:
                    locked_masked[key] = int(run.amax[b, p])
            K, V, z = snap[key]
            np.testing.assert_array_equal(run.K[:, b, :, p], K)
            np.testing.assert_array_equal(run.V[:, b, :, p], V)
            np.testing.assert_array_equal(run.prev_logits[key][0], z)
    assert len(locked_masked) > 3
    assert not (run.tokens == cfg.model.mask_id).any()
    positions = [p for _, _, p, _ in run.unmask_events]
    assert sorted(positions) == list(range(cfg.prompt_len, cfg.seq_len))     # each masked position once
    for (b, p), tok in locked_masked.items():
        assert run.tokens[b, p] == tok                                       # the argmax stored at lock time
    none = generate(cfg.replace(kl_eps=0.0, conf_tau=-1.0), tiny_w, tiny_tok)
    assert not none.lock.any()


def test_cb_dus_with_unreachable_bound_is_top1_decoding(tiny_w, tiny_tok):
    """A confidence bound no token reaches leaves only the forced best token per step: the
    generation is exactly top-1-confidence decoding."""
    a = generate(TINY.replace(unmask="cb_dus", cb_tau=2.0, tokens_per_step=4), tiny_w, tiny_tok)
    b = generate(TINY.replace(unmask="topconf", tokens_per_step=1), tiny_w, tiny_tok)
    np.testing.assert_array_equal(a.tokens, b.tokens)
    assert a.n_steps == b.n_steps == TINY.gen_len


def test_cb_dus_generation_unmasks_each_position_once(tiny_w, tiny_tok):
    cfg = TINY.replace(unmask="cb_dus", cb_tau=0.0, tokens_per_step=4)
    run = generate(cfg, tiny_w, tiny_tok)
    assert not (run.tokens == cfg.model.mask_id).any()
    positions = [p for _, _, p, _ in run.unmask_events]
    assert sorted(positions) == list(range(cfg.prompt_len, cfg.seq_len))
    by_step = {}
    for step, b, p, _ in run.unmask_events:
        by_step.setdefault(step, []).append(p)
    for ps in by_step.values():                                 # each step: non-adjacent, at most 4
        ps.sort()
        assert len(ps) <= 4 and all(q - p >= 2 for p, q in zip(ps, ps[1:]))
    assert run.n_steps < cfg.gen_len                            # several tokens per step on average


def test_es_skip_step_rewrites_only_recomputed_rows(tiny_w, tiny_tok):
    cfg = TINY
    run = OracleRun(cfg, tiny_w, tiny_tok)
    first = run.step()                             # refresh
    K0, V0 = run.K.copy(), run.V.copy()
    rec = run.step()                               # first skip step
    assert rec["kind"] == "skip" and rec["k"] == 8
    ls = cfg.skip_layer
    s, e = cfg.prompt_len, cfg.seq_len
    act = set(rec["rows"][1].tolist())
    assert len(act) == 8
    # layers below the skip layer: every candidate (block) row is rewritten, the prompt is not
    np.testing.assert_array_equal(run.K[:ls, :, :, :s], K0[:ls, :, :, :s])
    # (layer-0 K depends only on the row's own token, so the rows unmasked by the
    # refresh are the ones whose rewritten K differs)
    for _, p, _ in first["committed"]:
        assert np.any(run.K[0, 0, :, p] != K0[0, 0, :, p])
    # layers at and above it: only active rows change
    for p in range(cfg.seq_len):
        changed = np.any(run.K[ls:, 0, :, p] != K0[ls:, 0, :, p])
        if p not in act:
            assert not changed
    # the vocabulary projection ran only on active masked rows
    lm_pos = set(rec["rows"][1][rec["lm_rows"]].tolist())
    assert lm_pos <= act


def test_es_scores_follow_eq1_on_the_step(tiny_w, tiny_tok):
    # the step's scores equal Eq. 1 evaluated on the stored states it used
    run = OracleRun(TINY, tiny_w, tiny_tok)
    run.step()
    conf_before = run.conf.copy()
    masked_prev = run.masked_prev.copy()
    h_prev = run.h_prev.copy()
    rec = run.step()
    b, p = rec["cand"]
    c = np.where(masked_prev[b, p], conf_before[b, p], 0.0)
    d = TINY.model.d_model
    var = np.abs(rec["h_skip"] - h_prev[b, p]).sum(-1) / (np.sqrt(d) * np.linalg.norm(h_prev[b, p], axis=-1))
    np.testing.assert_allclose(rec["scores"], 0.5 * c + 0.5 * var, rtol=1e-12)


def test_batch_rows_are_independent(tiny_w):
    # two sequences in one batch evolve exactly as when each runs alone
    cfg = TINY.replace(batch=2)
    tok = make_tokens(cfg).numpy()
    both = generate(cfg, tiny_w, tok)
    for b in range(2):
        one = generate(TINY, tiny_w, tok[b:b + 1])
        np.testing.assert_array_equal(both.tokens[b], one.tokens[0])
        np.testing.assert_allclose(both.K[:, b], one.K[:, 0], rtol=1e-12, atol=1e-14)


def test_gqa_model_generates(tiny_w):
    cfg = scaled(TINY, n_heads=4, n_kv_heads=2)
    w = make_weights(cfg.model)
    run = generate(cfg.replace(policy="surelock"), w, make_tokens(cfg).numpy())
    assert not np.any(run.tokens == cfg.model.mask_id)

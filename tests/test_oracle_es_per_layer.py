"""Pins of the oracle's per-layer ES-dLLM re-selection (ES-dLLM summary sec. 2.1,
item 2: the top k is chosen at the start of each layer).

The per-layer skip step is pinned against the per-step one, which the step
pins already hold, in the cases where the two must agree exactly:

* one scored layer (skip layer = last layer) is the per-step step;
* alpha = 1 makes every layer's score the previous confidence alone, so every
  layer keeps the same rows, again the per-step step;
* keep ratio 1 over all rows is the full recompute.

The rest checks the parts that only the per-layer step has: Eq. 1 on each
layer's input, the cached output a skipped row carries into the next layer
(read back from an independent full pass), and K/V written only for the rows
chosen at that layer.
"""
import numpy as np
import pytest

from oracle.steps import OracleRun, generate
from synth import get_config, make_tokens, make_weights
from synth.configs import scaled

BASE = scaled(get_config("tiny"), n_layers=4)
PL = BASE.replace(es_per_layer=True, skip_layer=1)


@pytest.fixture(scope="module")
def w4():
    return make_weights(BASE.model)


@pytest.fixture(scope="module")
def tok():
    return make_tokens(BASE).numpy()


def _same_run(a, b):
    np.testing.assert_array_equal(a.tokens, b.tokens)
    np.testing.assert_array_equal(a.K, b.K)
    np.testing.assert_array_equal(a.V, b.V)
    np.testing.assert_array_equal(a.conf, b.conf)
    assert a.unmask_events == b.unmask_events


def test_one_scored_layer_is_the_per_step_choice(w4, tok):
    last = BASE.model.n_layers - 1
    _same_run(generate(PL.replace(skip_layer=last), w4, tok),
              generate(BASE.replace(skip_layer=last), w4, tok))


def test_confidence_only_scores_keep_the_same_rows_at_every_layer(w4, tok):
    a = generate(PL.replace(alpha=1.0), w4, tok)
    b = generate(BASE.replace(skip_layer=1, alpha=1.0), w4, tok)
    _same_run(a, b)


def test_keep_all_equals_full_recompute(w4, tok):
    a = generate(PL.replace(keep_ratio=1.0, cand_scope="all"), w4, tok)
    b = generate(BASE.replace(policy="vanilla"), w4, tok)
    _same_run(a, b)


def test_each_masked_position_unmasked_once(w4, tok):
    run = generate(PL, w4, tok)
    pos = [(b, p) for _, b, p, _ in run.unmask_events]
    assert len(pos) == len(set(pos)) == PL.batch * PL.gen_len
    assert not np.any(run.tokens == PL.model.mask_id)


def test_scores_follow_eq1_on_each_layer_input(w4, tok):
    run = OracleRun(PL, w4, tok)
    run.step()                                       # refresh
    conf0, masked0 = run.conf.copy(), run.masked_prev.copy()
    es_in0 = run.es_in.copy()
    rec = run.step()
    assert rec["kind"] == "skip"
    b, p = rec["cand"]
    c = np.where(masked0[b, p], conf0[b, p], 0.0)
    d, ls, a = PL.model.d_model, PL.skip_layer, PL.alpha
    for j, l in enumerate(range(ls, PL.model.n_layers)):
        x, prev = rec["layer_in"][j], es_in0[l][b, p]
        var = np.abs(x - prev).sum(-1) / (np.sqrt(d) * np.linalg.norm(prev, axis=-1))
        np.testing.assert_allclose(rec["layer_scores"][j], a * c + (1 - a) * var, rtol=1e-12, atol=0)
        if j:
            # a row the previous layer skipped enters with the state it had last iteration:
            # its variation term is exactly zero
            skipped = np.setdiff1d(np.arange(len(p)), rec["layer_active"][j - 1])
            np.testing.assert_array_equal(rec["layer_scores"][j][skipped], a * c[skipped])
        np.testing.assert_array_equal(run.es_in[l][b, p], x)


def test_skipped_row_carries_its_cached_output(w4, tok):
    """Forced choices: rows {0..7} at the skip layer, rows {4..11} at the next.  Rows 8..11
    enter the next layer with their skip-layer output of the refresh step (taken here from
    an independent full pass that keeps every layer's output); rows 4..7 with the output
    just computed, which is the layer applied to their inputs against the step's cache."""
    n = PL.block_len
    run = OracleRun(PL, w4, tok)
    run.step()
    ref = OracleRun(PL.replace(policy="dllm_cache", es_per_layer=False), w4, tok)
    ref.step()                                       # the same full pass, every output kept
    K0, V0 = run.K.copy(), run.V.copy()
    L, ls = PL.model.n_layers, PL.skip_layer
    forced = []
    for j in range(L - ls):
        s = np.zeros(n)
        s[(np.arange(8) + 4 * min(j, 1))] = 1.0      # j = 0: rows 0..7; j >= 1: rows 4..11
        forced.append(s)
    rec = run.step(forced_scores=forced)
    b, p = rec["cand"]
    np.testing.assert_array_equal(rec["layer_active"][0], np.arange(8))
    np.testing.assert_array_equal(rec["layer_active"][1], np.arange(4, 12))
    x1 = rec["layer_in"][1]
    for i in range(8, n):                            # skipped at the skip layer
        np.testing.assert_array_equal(x1[i], ref.h_cache[ls][b[i], p[i]])
    act = np.arange(8)
    Kc, Vc = K0[ls].copy(), V0[ls].copy()
    fresh = run.model.layer(ls, rec["layer_in"][0][act], b[act], p[act], Kc, Vc)
    np.testing.assert_array_equal(x1[act], fresh)


def test_kv_rewritten_only_for_rows_chosen_at_that_layer(w4, tok):
    # forced choices that differ from layer to layer: rows 4j .. 4j+7 at the j-th scored layer
    n = PL.block_len
    run = OracleRun(PL, w4, tok)
    run.step()
    K0 = run.K.copy()
    ls, L = PL.skip_layer, PL.model.n_layers
    forced = []
    for j in range(L - ls):
        s = np.zeros(n)
        s[4 * j + np.arange(8)] = 1.0
        forced.append(s)
    rec = run.step(forced_scores=forced)
    b, p = rec["cand"]
    for j, l in enumerate(range(ls, L)):
        chosen = p[rec["layer_active"][j]]
        np.testing.assert_array_equal(chosen, PL.prompt_len + 4 * j + np.arange(8))
        changed = {q for q in range(PL.seq_len) if np.any(run.K[l, 0, :, q] != K0[l, 0, :, q])}
        assert changed <= set(chosen.tolist())
    # the vocabulary projection covers the rows chosen at the last layer only
    assert set(rec["rows"][1][rec["lm_rows"]].tolist()) <= set(p[rec["layer_active"][-1]].tolist())

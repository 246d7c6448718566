"""ES-dLLM with the top k chosen again at every layer from the skip layer on
(ES-dLLM summary sec. 2.1, item 2), through the engine, against the oracle.

The step comparison is teacher-forced as in the per-step ES tests: at every
scored layer the engine takes the oracle's scores for that layer, and after
the step the oracle's tokens and confidences are written into the GPU state.
Checked per layer: the input every candidate enters the layer with (the carry
of a skipped row's cached output included), the Eq. 1 scores on the bf16 path,
the exact chosen rows; per step: outputs, confidences and every K/V cache row.
"""
import numpy as np
import pytest
import torch

from oracle.policy import es_importance, topk_select
from oracle.steps import OracleRun
from synth import get_config, make_tokens, make_weights
from synth.configs import scaled

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from token_skip_denoising_b200._lib import DllmError
    from token_skip_denoising_b200.engine import Engine, kernel_launches

DEV = "cuda"
BASE = scaled(get_config("tiny"), n_layers=4)
PL = BASE.replace(es_per_layer=True, skip_layer=1)
TOL_HIDDEN = 2e-2


TOL_SCORE = 1e-4     # Eq. 1 in fp32 on the GPU's own inputs


def _c_term(eng, flat):
    idx = torch.tensor(flat, device=DEV)
    return np.where(eng.buffer("masked_prev")[idx].cpu().numpy() != 0,
                    eng.buffer("conf")[idx].double().cpu().numpy(), 0.0)


def _prev_input(eng, l, ls, flat):
    """The GPU's record of each candidate's input of layer l in the last iteration."""
    idx = torch.tensor(flat, device=DEV)
    if l == ls:
        return eng.buffer("hprev")[idx].double().cpu().numpy()
    return eng.buffer("es_in")[l - ls - 1][idx].double().cpu().numpy()


def _rowrel(a, b):
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    return float((np.abs(a - b).max(1) / np.maximum(np.abs(b).max(1), 1e-30)).max())


@pytest.fixture(scope="module")
def w4():
    return make_weights(BASE.model)


def _dev(w):
    return {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in w.items()}


def _flat(b_idx, pos, N):
    return np.asarray(b_idx) * N + np.asarray(pos)


@pytest.mark.parametrize("layer_kernel", ["split", "fused"])
@pytest.mark.parametrize("batch", [1, 2])
def test_per_layer_steps_match_oracle_teacher_forced(w4, layer_kernel, batch):
    cfg = PL.replace(batch=batch)
    tok0 = make_tokens(cfg)
    orc = OracleRun(cfg, w4, tok0.numpy())
    eng = Engine(cfg, _dev(w4), tok0.to(DEV).contiguous(), layer_kernel=layer_kernel)
    N, L, ls, a = cfg.seq_len, cfg.model.n_layers, cfg.skip_layer, cfg.alpha
    kc, vc = eng.buffer("kcache"), eng.buffer("vcache")
    hid, conf, amax = eng.buffer("hidden"), eng.buffer("conf"), eng.buffer("argmax")
    n_skip = 0
    while not orc.done:
        rec = orc.step()
        kind = eng.begin_step()
        assert kind == ("full" if rec["kind"] == "refresh" else "skip")
        if kind == "skip":
            c_g = _c_term(eng, _flat(*rec["cand"], N))     # masked_prev rolls forward at the last layer
        for l in range(L):
            if l >= ls:
                if kind == "skip":
                    j = l - ls
                    flat = _flat(*rec["cand"], N)
                    prev = _prev_input(eng, l, ls, flat)
                    eng.select_active(torch.tensor(rec["layer_scores"][j], dtype=torch.float32, device=DEV))
                    # every candidate's input of this layer, skipped rows carrying their cached output
                    hx = hid[torch.tensor(flat, device=DEV)].cpu().numpy()
                    assert _rowrel(hx, rec["layer_in"][j]) < TOL_HIDDEN
                    gs = eng.buffer("scores")[:len(flat)].cpu().numpy().astype(np.float64)
                    ref = rec["layer_scores"][j]
                    # Eq. 1 element by element on the GPU's own input of this layer and its record of
                    # the previous iteration's
                    np.testing.assert_allclose(gs, es_importance(cfg.alpha, c_g, hx.astype(np.float64), prev),
                                               rtol=TOL_SCORE, atol=1e-7)
                    if j:
                        # rows the previous layer skipped: variation exactly zero, confidence term only
                        skipped = np.setdiff1d(np.arange(len(flat)), rec["layer_active"][j - 1])
                        np.testing.assert_allclose(gs[skipped], ref[skipped], rtol=1e-6, atol=1e-7)
                    nsel = int(eng.buffer("nrows")[0])
                    np.testing.assert_array_equal(eng.buffer("rows")[:nsel].cpu().numpy(),
                                                  flat[rec["layer_active"][j]])
                else:
                    eng.select_active()
            eng.layer_forward(l)
        rows = eng.buffer("rows")
        nrows = int(eng.buffer("nrows")[0])
        flat = _flat(*rec["rows"], N)
        np.testing.assert_array_equal(rows[:nrows].cpu().numpy(), flat)
        assert _rowrel(hid[torch.tensor(flat, device=DEV)].cpu().numpy(), rec["h_out"]) < TOL_HIDDEN
        eng.unmask()
        torch.cuda.synchronize()
        lm = flat[rec["lm_rows"]]
        np.testing.assert_allclose(conf[torch.tensor(lm, device=DEV)].cpu().numpy(), orc.conf.reshape(-1)[lm],
                                   rtol=5e-2, atol=1e-5)
        for l in range(L):
            assert _rowrel(kc[l].float().cpu().numpy().reshape(-1, cfg.model.head_dim),
                           orc.K[l].reshape(-1, cfg.model.head_dim)) < 2e-2
            assert _rowrel(vc[l].float().cpu().numpy().reshape(-1, cfg.model.head_dim),
                           orc.V[l].reshape(-1, cfg.model.head_dim)) < 2e-2
        n_skip += kind == "skip"
        eng.tokens.copy_(torch.tensor(orc.tokens, dtype=torch.int32))
        conf.copy_(torch.tensor(orc.conf.reshape(-1), dtype=torch.float32))
        amax.copy_(torch.tensor(orc.amax.reshape(-1), dtype=torch.int32))
    assert n_skip == 7
    assert eng.done


def test_forced_layer_choices_that_differ(w4):
    """Forced scores that pick rows 4j .. 4j+7 at the j-th scored layer: the engine keeps
    those rows at each layer and rewrites K/V only for them, as the oracle does."""
    cfg = PL
    tok0 = make_tokens(cfg)
    orc = OracleRun(cfg, w4, tok0.numpy())
    eng = Engine(cfg, _dev(w4), tok0.to(DEV).contiguous(), layer_kernel="split")
    orc.step()
    eng.step()
    eng.tokens.copy_(torch.tensor(orc.tokens, dtype=torch.int32))
    eng.buffer("conf").copy_(torch.tensor(orc.conf.reshape(-1), dtype=torch.float32))
    eng.buffer("argmax").copy_(torch.tensor(orc.amax.reshape(-1), dtype=torch.int32))
    L, ls, n, N = cfg.model.n_layers, cfg.skip_layer, cfg.block_len, cfg.seq_len
    forced = []
    for j in range(L - ls):
        s = np.zeros(n)
        s[4 * j + np.arange(8)] = 1.0
        forced.append(s)
    rec = orc.step(forced_scores=forced)
    k0 = eng.buffer("kcache").clone()
    assert eng.begin_step() == "skip"
    hid = eng.buffer("hidden")
    for l in range(L):
        if l >= ls:
            eng.select_active(torch.tensor(forced[l - ls], dtype=torch.float32, device=DEV))
            flat = _flat(*rec["cand"], N)
            hx = hid[torch.tensor(flat, device=DEV)].cpu().numpy()
            assert _rowrel(hx, rec["layer_in"][l - ls]) < TOL_HIDDEN
        eng.layer_forward(l)
    eng.unmask()
    torch.cuda.synchronize()
    k1 = eng.buffer("kcache")
    for j, l in enumerate(range(ls, L)):
        chosen = cfg.prompt_len + 4 * j + np.arange(8)
        changed = (k1[l] != k0[l]).any(dim=-1).any(dim=1)[0].cpu().numpy()
        assert set(np.nonzero(changed)[0].tolist()) <= set(chosen.tolist())
        assert _rowrel(k1[l].float().cpu().numpy().reshape(-1, cfg.model.head_dim),
                       orc.K[l].reshape(-1, cfg.model.head_dim)) < 2e-2


@pytest.mark.parametrize("batch", [1, 2])
def test_fused_per_layer_run_matches_oracle_teacher_forced(w4, batch):
    """dllm_select_layers_forward: on skip steps one persistent launch scores and chooses the
    rows at the start of every layer itself.  With the oracle's per-layer scores forced, the
    chosen rows are exact and outputs, confidences and caches agree within tolerance; the
    scores it computes (the last layer's are kept) agree element by element with Eq. 1 evaluated
    on the GPU's own inputs of that layer."""
    cfg = PL.replace(batch=batch)
    tok0 = make_tokens(cfg)
    orc = OracleRun(cfg, w4, tok0.numpy())
    eng = Engine(cfg, _dev(w4), tok0.to(DEV).contiguous())
    N, L, ls = cfg.seq_len, cfg.model.n_layers, cfg.skip_layer
    kc, vc = eng.buffer("kcache"), eng.buffer("vcache")
    hid, conf, amax = eng.buffer("hidden"), eng.buffer("conf"), eng.buffer("argmax")
    n_skip = 0
    while not orc.done:
        rec = orc.step()
        kind = eng.begin_step()
        eng.layers_forward(0, ls)
        forced = None
        if kind == "skip":
            forced = torch.tensor(np.stack(rec["layer_scores"]), dtype=torch.float32, device=DEV).contiguous()
            cflat = _flat(*rec["cand"], N)
            c_g = _c_term(eng, cflat)
            prev_last = _prev_input(eng, L - 1, ls, cflat)
        torch.cuda.synchronize()
        n0 = kernel_launches()
        eng.select_layers_forward(forced)
        torch.cuda.synchronize()
        if kind == "skip":
            assert kernel_launches() - n0 == 2            # the row counts, then one fused launch
            gs = eng.buffer("scores")[:len(rec["cand"][0])].cpu().numpy().astype(np.float64)
            # the last layer's in-kernel Eq. 1, element by element: its input is what the run left in
            # the per-layer record, the previous iteration's what the record held before the run
            cur_last = _prev_input(eng, L - 1, ls, cflat)
            np.testing.assert_allclose(gs, es_importance(cfg.alpha, c_g, cur_last, prev_last),
                                       rtol=TOL_SCORE, atol=1e-7)
            assert _rowrel(cur_last, rec["layer_in"][-1]) < TOL_HIDDEN
            n_skip += 1
        rows = eng.buffer("rows")
        nrows = int(eng.buffer("nrows")[0])
        flat = _flat(*rec["rows"], N)
        np.testing.assert_array_equal(rows[:nrows].cpu().numpy(), flat)
        assert _rowrel(hid[torch.tensor(flat, device=DEV)].cpu().numpy(), rec["h_out"]) < TOL_HIDDEN
        eng.unmask()
        torch.cuda.synchronize()
        lm = flat[rec["lm_rows"]]
        np.testing.assert_allclose(conf[torch.tensor(lm, device=DEV)].cpu().numpy(), orc.conf.reshape(-1)[lm],
                                   rtol=5e-2, atol=1e-5)
        for l in range(L):
            assert _rowrel(kc[l].float().cpu().numpy().reshape(-1, cfg.model.head_dim),
                           orc.K[l].reshape(-1, cfg.model.head_dim)) < 2e-2
            assert _rowrel(vc[l].float().cpu().numpy().reshape(-1, cfg.model.head_dim),
                           orc.V[l].reshape(-1, cfg.model.head_dim)) < 2e-2
        eng.tokens.copy_(torch.tensor(orc.tokens, dtype=torch.int32))
        conf.copy_(torch.tensor(orc.conf.reshape(-1), dtype=torch.float32))
        amax.copy_(torch.tensor(orc.amax.reshape(-1), dtype=torch.int32))
    assert n_skip == 7
    assert eng.done


def test_fused_per_layer_run_with_differing_forced_choices(w4):
    """Forced choices that move from layer to layer (rows 4j .. 4j+7 at the j-th scored layer)
    through the in-kernel choice: the same rows, inputs carried the same way as the oracle."""
    cfg = PL
    tok0 = make_tokens(cfg)
    orc = OracleRun(cfg, w4, tok0.numpy())
    eng = Engine(cfg, _dev(w4), tok0.to(DEV).contiguous())
    orc.step()
    eng.step()
    eng.tokens.copy_(torch.tensor(orc.tokens, dtype=torch.int32))
    eng.buffer("conf").copy_(torch.tensor(orc.conf.reshape(-1), dtype=torch.float32))
    eng.buffer("argmax").copy_(torch.tensor(orc.amax.reshape(-1), dtype=torch.int32))
    L, ls, n, N = cfg.model.n_layers, cfg.skip_layer, cfg.block_len, cfg.seq_len
    forced = np.zeros((L - ls, n))
    for j in range(L - ls):
        forced[j, 4 * j + np.arange(8)] = 1.0
    rec = orc.step(forced_scores=list(forced))
    k0 = eng.buffer("kcache").clone()
    assert eng.begin_step() == "skip"
    eng.layers_forward(0, ls)
    eng.select_layers_forward(torch.tensor(forced, dtype=torch.float32, device=DEV).contiguous())
    flat = _flat(*rec["rows"], N)
    np.testing.assert_array_equal(eng.buffer("rows")[:8].cpu().numpy(), flat)
    assert _rowrel(eng.buffer("hidden")[torch.tensor(flat, device=DEV)].cpu().numpy(), rec["h_out"]) < TOL_HIDDEN
    eng.unmask()
    torch.cuda.synchronize()
    k1 = eng.buffer("kcache")
    for j, l in enumerate(range(ls, L)):
        chosen = cfg.prompt_len + 4 * j + np.arange(8)
        changed = (k1[l] != k0[l]).any(dim=-1).any(dim=1)[0].cpu().numpy()
        assert set(np.nonzero(changed)[0].tolist()) <= set(chosen.tolist())
        assert _rowrel(k1[l].float().cpu().numpy().reshape(-1, cfg.model.head_dim),
                       orc.K[l].reshape(-1, cfg.model.head_dim)) < 2e-2


@pytest.mark.parametrize("batch", [1, 2])
def test_fused_per_layer_choice_on_its_own_scores_is_the_top_k(w4, batch):
    """No teacher forcing: after each fused per-layer run, the last layer's scores match Eq. 1
    on the GPU's own inputs of that layer and the rows it kept are the top k of those scores,
    bit for bit."""
    cfg = PL.replace(batch=batch)
    eng = Engine(cfg, _dev(w4), make_tokens(cfg).to(DEV).contiguous())
    N, L, ls, n = cfg.seq_len, cfg.model.n_layers, cfg.skip_layer, cfg.block_len
    k = cfg.keep_count(n)
    n_skip = 0
    while not eng.done:
        kind = eng.begin_step()
        eng.layers_forward(0, ls)
        if kind == "skip":
            s0 = cfg.prompt_len + eng.progress()["block"] * cfg.block_len
            cflat = np.concatenate([b * N + s0 + np.arange(n) for b in range(cfg.batch)])
            c_g = _c_term(eng, cflat)
            prev_last = _prev_input(eng, L - 1, ls, cflat)
        eng.select_layers_forward()
        torch.cuda.synchronize()
        if kind == "skip":
            gs = eng.buffer("scores")[:cfg.batch * n].cpu().numpy().astype(np.float64)
            cur_last = _prev_input(eng, L - 1, ls, cflat)
            np.testing.assert_allclose(gs, es_importance(cfg.alpha, c_g, cur_last, prev_last),
                                       rtol=TOL_SCORE, atol=1e-7)
            want = np.concatenate([b * N + s0 + topk_select(gs[b * n:(b + 1) * n], k) for b in range(cfg.batch)])
            np.testing.assert_array_equal(eng.buffer("rows")[:cfg.batch * k].cpu().numpy(), want)
            n_skip += 1
        eng.unmask()
    assert n_skip == 7


def test_keep_all_per_layer_equals_vanilla(w4):
    tok0 = make_tokens(BASE)
    a = Engine(PL.replace(keep_ratio=1.0, cand_scope="all"), _dev(w4), tok0.to(DEV).contiguous(),
               layer_kernel="split")
    b = Engine(BASE.replace(policy="vanilla"), _dev(w4), tok0.to(DEV).contiguous(), layer_kernel="split")
    a.generate()
    b.generate()
    torch.cuda.synchronize()
    assert torch.equal(a.tokens, b.tokens)
    assert torch.equal(a.buffer("kcache"), b.buffer("kcache"))
    assert torch.equal(a.buffer("vcache"), b.buffer("vcache"))


@pytest.mark.parametrize("batch", [1, 2])
def test_per_layer_generation_unmasks_each_position_once(w4, batch):
    cfg = PL.replace(batch=batch)
    tok0 = make_tokens(cfg)
    eng = Engine(cfg, _dev(w4), tok0.to(DEV).contiguous())
    steps = 0
    while not eng.done:
        info = eng.step(info=True)
        if info["kind_name"] == "skip":
            assert info["rows_last"] == batch * cfg.keep_count(cfg.block_len)
        steps += 1
    tok = eng.tokens.cpu().numpy()
    assert steps == cfg.gen_len // cfg.tokens_per_step
    assert not np.any(tok == cfg.model.mask_id)
    np.testing.assert_array_equal(tok[:, :cfg.prompt_len], tok0.numpy()[:, :cfg.prompt_len])


def test_out_of_order_calls_are_refused(w4):
    cfg = PL
    eng = Engine(cfg, _dev(w4), make_tokens(cfg).to(DEV).contiguous())
    eng.begin_step()
    eng.layers_forward(0, cfg.skip_layer)
    with pytest.raises(DllmError):
        eng.layer_forward(cfg.skip_layer)            # no select_active for this layer yet
    eng.select_active()
    with pytest.raises(DllmError):
        eng.layers_forward(cfg.skip_layer, cfg.model.n_layers)   # more than one layer at once
    with pytest.raises(DllmError):
        eng.unmask()                                 # layers left
    with pytest.raises(DllmError):
        eng.select_layers_forward()                  # a per-layer call was made in this step

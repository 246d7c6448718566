"""Whole denoising steps through the engine (dllm_begin_step / dllm_layer_forward /
dllm_select_active / dllm_unmask / dllm_step) against the oracle.

End-to-end trajectories of a bf16 path and an fp64 oracle part at near-tied
confidences, so the step-level comparison is teacher-forced: the oracle runs
the step first, the GPU step takes the oracle's selection scores, and after
the step the oracle's tokens and confidences are written into the GPU state.
"""
import numpy as np
import pytest
import torch

from oracle.policy import es_importance, topk_select
from oracle.steps import OracleRun
from synth import get_config, make_tokens, make_weights

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from token_skip_denoising_b200.engine import Engine, kernel_launches

DEV = "cuda"
TINY = get_config("tiny")
TOL_HIDDEN = 2e-2


TOL_SCORE = 1e-4     # Eq. 1 in fp32 on the GPU's own inputs: relative to each score


def _eq1_inputs(eng, flat):
    """The GPU's own Eq. 1 inputs for the candidate rows `flat`: current hidden state at the
    skip layer, the snapshot of the previous iteration, and c = conf if the row was masked at
    the start of the previous step, else 0."""
    idx = torch.tensor(flat, device=DEV)
    h = eng.buffer("hidden")[idx].double().cpu().numpy()
    hp = eng.buffer("hprev")[idx].double().cpu().numpy()
    c = np.where(eng.buffer("masked_prev")[idx].cpu().numpy() != 0, eng.buffer("conf")[idx].double().cpu().numpy(),
                 0.0)
    return h, hp, c


def _assert_scores(gs, want):
    np.testing.assert_allclose(gs, want, rtol=TOL_SCORE, atol=1e-7)


def _rowrel(a, b):
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    return float((np.abs(a - b).max(1) / np.maximum(np.abs(b).max(1), 1e-30)).max())


@pytest.fixture(scope="module")
def tiny_w_cpu():
    return make_weights(TINY.model)


def _to_dev(w):
    return {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in w.items()}


def _flat(b_idx, pos, N):
    return np.asarray(b_idx) * N + np.asarray(pos)


def _engine(cfg, w, tokens, **over):
    return Engine(cfg, _to_dev(w), tokens.to(DEV).contiguous(), **over)


@pytest.mark.parametrize("cfg", [TINY, TINY.replace(batch=2), TINY.replace(policy="vanilla"),
                                 TINY.replace(tokens_per_step=1, block_len=8)])
def test_generation_unmasks_each_position_once(cfg, tiny_w_cpu):
    tok0 = make_tokens(cfg)
    eng = _engine(cfg, tiny_w_cpu, tok0)
    seen = np.zeros((cfg.batch, cfg.seq_len), int)
    steps = 0
    width = cfg.tokens_per_step                     # pos_out / tok_out are [B, n] for top-n unmasking
    pos = torch.full((cfg.batch, width), -1, dtype=torch.int32, device=DEV)
    tk = torch.full((cfg.batch, width), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(cfg.batch, dtype=torch.int32, device=DEV)
    while not eng.done:
        eng.begin_step()
        ls = cfg.skip_layer if cfg.policy == "es" else cfg.model.n_layers
        for l in range(cfg.model.n_layers):
            if l == ls:
                eng.select_active()
            eng.layer_forward(l)
        eng.unmask(pos, tk, cnt)
        for b in range(cfg.batch):
            for i in range(int(cnt[b])):
                seen[b, int(pos[b, i])] += 1
        steps += 1
    tok = eng.tokens.cpu().numpy()
    assert steps == cfg.gen_len // cfg.tokens_per_step
    assert np.all(seen[:, cfg.prompt_len:] == 1) and np.all(seen[:, :cfg.prompt_len] == 0)
    assert not np.any(tok == cfg.model.mask_id)
    np.testing.assert_array_equal(tok[:, :cfg.prompt_len], tok0.numpy()[:, :cfg.prompt_len])


def test_es_steps_match_oracle_teacher_forced(tiny_w_cpu):
    cfg = TINY
    tok0 = make_tokens(cfg)
    orc = OracleRun(cfg, tiny_w_cpu, tok0.numpy())
    eng = _engine(cfg, tiny_w_cpu, tok0)
    N, L, ls = cfg.seq_len, cfg.model.n_layers, cfg.skip_layer
    kc, vc = eng.buffer("kcache"), eng.buffer("vcache")
    hid, conf, amax = eng.buffer("hidden"), eng.buffer("conf"), eng.buffer("argmax")
    n_skip = 0
    while not orc.done:
        rec = orc.step()
        kind = eng.begin_step()
        assert kind == ("full" if rec["kind"] == "refresh" else "skip")
        for l in range(L):
            if l == ls:
                if kind == "skip":
                    b_idx, pos = rec["cand"]
                    # hidden state of the candidates at the skip layer (Eq. 1 input)
                    hc = hid[torch.tensor(_flat(b_idx, pos, N), device=DEV)].cpu().numpy()
                    assert _rowrel(hc, rec["h_skip"]) < TOL_HIDDEN
                    h_g, hp_g, c_g = _eq1_inputs(eng, _flat(b_idx, pos, N))
                    forced = torch.tensor(rec["scores"], dtype=torch.float32, device=DEV)
                    eng.select_active(forced)
                    gpu_scores = eng.buffer("scores")[:len(rec["scores"])].double().cpu().numpy()
                    # Eq. 1 element by element on the GPU's own inputs
                    _assert_scores(gpu_scores, es_importance(cfg.alpha, c_g, h_g, hp_g))
                    n_skip += 1
                else:
                    eng.select_active()
            eng.layer_forward(l)
        rows = eng.buffer("rows")
        nrows = int(eng.buffer("nrows")[0])
        flat = _flat(*rec["rows"], N)
        np.testing.assert_array_equal(rows[:nrows].cpu().numpy(), flat)      # same active set, bit-exact
        assert _rowrel(hid[torch.tensor(flat, device=DEV)].cpu().numpy(), rec["h_out"]) < TOL_HIDDEN
        eng.unmask()
        torch.cuda.synchronize()
        lm = flat[rec["lm_rows"]]
        np.testing.assert_allclose(conf[torch.tensor(lm, device=DEV)].cpu().numpy(), orc.conf.reshape(-1)[lm],
                                   rtol=5e-2, atol=1e-5)
        # caches: every layer, every row the oracle holds
        for l in range(L):
            assert _rowrel(kc[l].float().cpu().numpy().reshape(-1, cfg.model.head_dim),
                           orc.K[l].reshape(-1, cfg.model.head_dim)) < 2e-2
        # teacher forcing of the decisions
        eng.tokens.copy_(torch.tensor(orc.tokens, dtype=torch.int32))
        conf.copy_(torch.tensor(orc.conf.reshape(-1), dtype=torch.float32))
        amax.copy_(torch.tensor(orc.amax.reshape(-1), dtype=torch.int32))
    assert n_skip == 7
    assert eng.done


@pytest.mark.parametrize("batch", [1, 2])
def test_es_choice_inside_the_fused_run_teacher_forced(tiny_w_cpu, batch):
    """dllm_select_layers_forward on a skip step: one persistent launch scores the candidates
    by Eq. 1, keeps the top k of each sequence and runs the remaining layers on them.  With the
    oracle's scores forced the kept rows are exact; its own Eq. 1 scores, the outputs, the
    confidences and the caches agree with the oracle within tolerance."""
    cfg = TINY.replace(batch=batch)
    tok0 = make_tokens(cfg)
    orc = OracleRun(cfg, tiny_w_cpu, tok0.numpy())
    eng = _engine(cfg, tiny_w_cpu, tok0)
    N, L, ls = cfg.seq_len, cfg.model.n_layers, cfg.skip_layer
    kc = eng.buffer("kcache")
    hid, conf, amax = eng.buffer("hidden"), eng.buffer("conf"), eng.buffer("argmax")
    n_skip = 0
    while not orc.done:
        rec = orc.step()
        kind = eng.begin_step()
        eng.layers_forward(0, ls)
        forced = None
        if kind == "skip":
            forced = torch.tensor(rec["scores"][None], dtype=torch.float32, device=DEV).contiguous()
            h_g, hp_g, c_g = _eq1_inputs(eng, _flat(*rec["cand"], N))
        torch.cuda.synchronize()
        n0 = kernel_launches()
        eng.select_layers_forward(forced)
        torch.cuda.synchronize()
        if kind == "skip":
            assert kernel_launches() - n0 == 2            # the row counts, then one fused launch
            gs = eng.buffer("scores")[:len(rec["scores"])].cpu().numpy().astype(np.float64)
            # the in-kernel Eq. 1, element by element on the GPU's own inputs
            _assert_scores(gs, es_importance(cfg.alpha, c_g, h_g, hp_g))
            n_skip += 1
        nrows = int(eng.buffer("nrows")[0])
        flat = _flat(*rec["rows"], N)
        np.testing.assert_array_equal(eng.buffer("rows")[:nrows].cpu().numpy(), flat)
        assert _rowrel(hid[torch.tensor(flat, device=DEV)].cpu().numpy(), rec["h_out"]) < TOL_HIDDEN
        eng.unmask()
        torch.cuda.synchronize()
        lm = flat[rec["lm_rows"]]
        np.testing.assert_allclose(conf[torch.tensor(lm, device=DEV)].cpu().numpy(), orc.conf.reshape(-1)[lm],
                                   rtol=5e-2, atol=1e-5)
        for l in range(L):
            assert _rowrel(kc[l].float().cpu().numpy().reshape(-1, cfg.model.head_dim),
                           orc.K[l].reshape(-1, cfg.model.head_dim)) < 2e-2
        eng.tokens.copy_(torch.tensor(orc.tokens, dtype=torch.int32))
        conf.copy_(torch.tensor(orc.conf.reshape(-1), dtype=torch.float32))
        amax.copy_(torch.tensor(orc.amax.reshape(-1), dtype=torch.int32))
    assert n_skip == 7
    assert eng.done


@pytest.mark.parametrize("path", ["fused", "split"])
@pytest.mark.parametrize("batch", [1, 2])
def test_es_choice_on_its_own_scores_is_the_top_k(tiny_w_cpu, path, batch):
    """No teacher forcing: on every skip step the GPU's Eq. 1 scores match Eq. 1 evaluated on
    the GPU's own inputs, and the kept rows are exactly the top k of those scores (ties to the
    lower position), bit for bit: the in-kernel rank count of the fused run, and the radix
    select of the split path."""
    cfg = TINY.replace(batch=batch)
    eng = _engine(cfg, tiny_w_cpu, make_tokens(cfg), layer_kernel=path)
    N, ls, n = cfg.seq_len, cfg.skip_layer, cfg.block_len
    k = cfg.keep_count(n)
    n_skip = 0
    while not eng.done:
        kind = eng.begin_step()
        eng.layers_forward(0, ls)
        if kind == "skip":
            s0 = cfg.prompt_len + eng.progress()["block"] * cfg.block_len
            flat = np.concatenate([b * N + s0 + np.arange(n) for b in range(cfg.batch)])
            h_g, hp_g, c_g = _eq1_inputs(eng, flat)
        if path == "fused":
            eng.select_layers_forward()
        else:
            eng.select_active()
            eng.layers_forward(ls, cfg.model.n_layers)
        torch.cuda.synchronize()
        if kind == "skip":
            gs = eng.buffer("scores")[:cfg.batch * n].cpu().numpy().astype(np.float64)
            _assert_scores(gs, es_importance(cfg.alpha, c_g, h_g, hp_g))
            want = np.concatenate([b * N + s0 + topk_select(gs[b * n:(b + 1) * n], k)
                                   for b in range(cfg.batch)])
            nrows = int(eng.buffer("nrows")[0])
            np.testing.assert_array_equal(eng.buffer("rows")[:nrows].cpu().numpy(), want)
            n_skip += 1
        eng.unmask()
    assert n_skip == 7


def test_keep_all_equals_vanilla_on_gpu(tiny_w_cpu):
    """keep ratio 1 over all rows is the full recompute, bit for bit, on the kernel-per-step
    layer (the fused layer's fp32 reductions are order-dependent, so it is held to the
    tolerances of the oracle comparisons instead)."""
    tok0 = make_tokens(TINY)
    a = _engine(TINY.replace(keep_ratio=1.0, cand_scope="all"), tiny_w_cpu, tok0, layer_kernel="split")
    b = _engine(TINY.replace(policy="vanilla"), tiny_w_cpu, tok0, layer_kernel="split")
    a.generate()
    b.generate()
    torch.cuda.synchronize()
    assert torch.equal(a.tokens, b.tokens)
    assert torch.equal(a.buffer("kcache"), b.buffer("kcache"))
    assert torch.equal(a.buffer("vcache"), b.buffer("vcache"))


def test_skip_step_rewrites_only_active_rows(tiny_w_cpu):
    cfg = TINY
    eng = _engine(cfg, tiny_w_cpu, make_tokens(cfg))
    eng.step()                                      # refresh
    torch.cuda.synchronize()
    k0, v0 = eng.buffer("kcache").clone(), eng.buffer("vcache").clone()
    info = eng.step(info=True)                      # skip step
    assert info["kind_name"] == "skip" and info["rows_first"] == 32 and info["rows_last"] == 8
    act = eng.buffer("rows")[:8].cpu().numpy()
    k1, v1 = eng.buffer("kcache"), eng.buffer("vcache")
    ls = cfg.skip_layer
    changed = (k1[ls:] != k0[ls:]).any(dim=-1).any(dim=0).any(dim=1)[0].cpu().numpy()   # [N]
    assert set(np.nonzero(changed)[0]) <= set(act.tolist())
    # the prompt is never rewritten in a skip step, at any layer
    assert torch.equal(k1[:, :, :, :cfg.prompt_len], k0[:, :, :, :cfg.prompt_len])
    assert torch.equal(v1[:, :, :, :cfg.prompt_len], v0[:, :, :, :cfg.prompt_len])
    assert info["lm_rows"] <= 8

"""The SureLock and dLLM-Cache step paths of the engine, and DUS unmasking, against the oracle.

SureLock runs with a seeded lock pattern (the measurement mode) so that locks
are decided without floating-point thresholds and the active sets can be
compared bit for bit; dLLM-Cache is compared with every response row selected
(tau = inf, rho = 1) for the same reason, and its cosine scores are compared
per layer within tolerance.  Decisions are teacher-forced as in the ES tests.
"""
import math

import numpy as np
import pytest
import torch

from oracle.policy import cosine_rows, dus_schedule, kl_from_logits, threshold_cap_select
from oracle.steps import OracleRun
from synth import get_config, make_tokens, make_weights

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from token_skip_denoising_b200.engine import Engine

DEV = "cuda"
TINY = get_config("tiny")
TOL_HIDDEN = 2e-2


def _rowrel(a, b):
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    return float((np.abs(a - b).max(1) / np.maximum(np.abs(b).max(1), 1e-30)).max())


@pytest.fixture(scope="module")
def tiny_w():
    return make_weights(TINY.model)


def _dev(w):
    return {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in w.items()}


def _force(eng, orc):
    eng.tokens.copy_(torch.tensor(orc.tokens, dtype=torch.int32))
    eng.buffer("conf").copy_(torch.tensor(orc.conf.reshape(-1), dtype=torch.float32))
    eng.buffer("argmax").copy_(torch.tensor(orc.amax.reshape(-1), dtype=torch.int32))


# ------------------------------------------------------------------ SureLock

@pytest.mark.parametrize("lock_masked", [False, True])
def test_surelock_steps_match_oracle_with_lock_pattern(tiny_w, lock_masked):
    cfg = TINY.replace(policy="surelock", tokens_per_step=2, batch=2, lock_masked=lock_masked)
    N = cfg.seq_len
    tok0 = make_tokens(cfg)
    pattern = np.zeros((cfg.batch, N), bool)
    pattern[:, ::3] = True
    pattern[1, 1::5] = True
    orc = OracleRun(cfg, tiny_w, tok0.numpy(), lock_pattern=pattern)
    eng = Engine(cfg, _dev(tiny_w), tok0.to(DEV).contiguous())
    pat_dev = torch.tensor(pattern.astype(np.uint8), device=DEV)
    eng.set_lock_pattern(pat_dev)
    hid = eng.buffer("hidden")
    locked_max = 0
    while not orc.done:
        rec = orc.step()
        info = eng.step(info=True)
        assert info["kind_name"] == "locked"
        flat = rec["rows"][0] * N + rec["rows"][1]
        nrows = int(eng.buffer("nrows")[0])
        np.testing.assert_array_equal(eng.buffer("rows")[:nrows].cpu().numpy(), flat)   # same active set
        assert _rowrel(hid[torch.tensor(flat, device=DEV)].cpu().numpy(), rec["h_out"]) < TOL_HIDDEN
        np.testing.assert_array_equal(eng.buffer("lock").cpu().numpy().reshape(cfg.batch, N),
                                      orc.lock.astype(np.uint8))
        # KL of the eligible rows that had a previous distribution: present exactly where the
        # oracle has one, and equal to KL(p_t || p_t-1) of the GPU's own two stored bf16 logit rows
        n_lm = int(eng.buffer("nlmrows")[0])
        assert n_lm == len(rec["lm_rows"])
        kl_g = eng.buffer("kl")[:n_lm].cpu().numpy().astype(np.float64)
        ok = ~np.isnan(rec["kl"])            # the oracle's: eligible rows with a previous distribution
        assert not np.isnan(kl_g[ok]).any()  # (the GPU also reports it for masked rows that have one)
        has = ~np.isnan(kl_g)
        if has.any():
            _check_kl_on_own_logits(eng, info["step"], eng.buffer("lmrows")[:n_lm].cpu().numpy()[has], kl_g[has])
        lm = flat[rec["lm_rows"]]
        np.testing.assert_allclose(eng.buffer("conf")[torch.tensor(lm, device=DEV)].cpu().numpy(),
                                   orc.conf.reshape(-1)[lm], rtol=5e-2, atol=1e-5)
        locked_max = max(locked_max, int(orc.lock.sum()))
        _force(eng, orc)
    assert locked_max > 10 and eng.done


TOL_KL_REL, TOL_KL_ABS = 1e-3, 1e-5     # well below the lock threshold eps = 1e-3


def _check_kl_on_own_logits(eng, step, flat, kl_gpu):
    """KL(p_t || p_t-1) in fp64 from the bf16 logits the GPU stored at steps t and t-1."""
    z = eng.buffer("zstore")
    cur = z[step & 1][torch.tensor(flat, device=DEV)].double().cpu().numpy()
    prv = z[(step + 1) & 1][torch.tensor(flat, device=DEV)].double().cpu().numpy()

    def lse(a):
        mx = a.max(1, keepdims=True)
        return (mx + np.log(np.exp(a - mx).sum(1, keepdims=True)))[:, 0]
    want = kl_from_logits(cur, lse(cur), prv, lse(prv))
    np.testing.assert_allclose(kl_gpu, want, rtol=TOL_KL_REL, atol=TOL_KL_ABS)


@pytest.mark.parametrize("lock_masked", [False, True])
def test_surelock_kl_rule_decisions(tiny_w, lock_masked):
    """The lock rule itself (no pattern), teacher-forced on the oracle's tokens:
    * kl_eps = 1e30, conf_tau = -1 makes the rule true wherever a KL exists, so the locks do not
      depend on floating point: the GPU's lock flags equal the oracle's at every step;
    * kl_eps = 1e-3: every LM row's decision equals "KL < eps and conf > tau" on the GPU's own
      KL and confidence (the decision is taken in the kernel's fp32 on both sides), and the KL
      equals fp64 KL of the GPU's stored logits to 1e-3 relative / 1e-5 absolute."""
    for eps, tau in ((1e30, -1.0), (1e-3, -1.0)):
        cfg = TINY.replace(policy="surelock", tokens_per_step=2, kl_eps=eps, conf_tau=tau, lock_masked=lock_masked)
        N = cfg.seq_len
        tok0 = make_tokens(cfg)
        orc = OracleRun(cfg, tiny_w, tok0.numpy())
        eng = Engine(cfg, _dev(tiny_w), tok0.to(DEV).contiguous())
        n_new = 0
        while not orc.done:
            lock0 = eng.buffer("lock").cpu().numpy().copy()
            tok_before = eng.tokens.cpu().numpy().reshape(-1).copy()
            orc.step()
            info = eng.step(info=True)
            lock1 = eng.buffer("lock").cpu().numpy()
            n_lm = int(eng.buffer("nlmrows")[0])
            flat = eng.buffer("lmrows")[:n_lm].cpu().numpy()
            kl_g = eng.buffer("kl")[:n_lm].cpu().numpy()
            conf_g = eng.buffer("conf")[torch.tensor(flat, device=DEV)].cpu().numpy()
            has = ~np.isnan(kl_g)
            if has.any():
                _check_kl_on_own_logits(eng, info["step"], flat[has], kl_g[has].astype(np.float64))
            if eps > 1e29:
                np.testing.assert_array_equal(lock1.reshape(cfg.batch, N), orc.lock.astype(np.uint8))
            else:
                eligible = np.ones(n_lm, bool) if lock_masked else tok_before[flat] != cfg.model.mask_id
                rule = eligible & has & (kl_g < np.float32(eps)) & (conf_g > np.float32(tau))
                np.testing.assert_array_equal(lock1[flat] != 0, (lock0[flat] != 0) | rule)
            n_new += int((lock1 != lock0).sum())
            _force(eng, orc)
            eng.buffer("lock").copy_(torch.tensor(orc.lock.reshape(-1).astype(np.uint8)))
        if eps > 1e29:
            assert n_new > 10


def test_surelock_eps_zero_never_locks(tiny_w):
    cfg = TINY.replace(policy="surelock", kl_eps=0.0, conf_tau=-1.0)
    eng = Engine(cfg, _dev(tiny_w), make_tokens(cfg).to(DEV).contiguous())
    while not eng.done:
        info = eng.step(info=True)
        assert info["rows_last"] == cfg.seq_len            # every row recomputed every step
    assert int(eng.buffer("lock").sum()) == 0
    assert not bool((eng.tokens == cfg.model.mask_id).any())


# ------------------------------------------------------------------ dLLM-Cache + DUS

def test_dllm_cache_full_selection_matches_oracle(tiny_w):
    cfg = TINY.replace(policy="dllm_cache", unmask="dus", block_len=8, prompt_interval=5,
                       sim_tau=float("inf"), rho_cap=1.0)
    N, L = cfg.seq_len, cfg.model.n_layers
    tok0 = make_tokens(cfg)
    orc = OracleRun(cfg, tiny_w, tok0.numpy())
    eng = Engine(cfg, _dev(tiny_w), tok0.to(DEV).contiguous())
    hcache = eng.buffer("hcache")
    n_partial = 0
    while not orc.done:
        rec = orc.step()
        kind = eng.begin_step()
        assert kind == ("full" if rec["kind"] == "refresh" else "partial")
        for l in range(L):
            eng.layer_forward(l)
            if kind == "partial":
                sims = eng.buffer("scores")[:cfg.batch * cfg.gen_len].cpu().numpy()
                ref = rec["layers"][l]["sims"]
                assert np.abs(sims - ref).max() < 2e-2
        eng.unmask()
        torch.cuda.synchronize()
        b_idx, pos = rec["rows"]
        flat = b_idx * N + pos
        got = hcache[L - 1][torch.tensor(flat, device=DEV)].cpu().numpy()
        assert _rowrel(got, rec["h_out"]) < TOL_HIDDEN
        n_partial += kind == "partial"
        _force(eng, orc)
    assert n_partial > 0 and eng.done


def _check_cos_on_own_values(eng, cfg, vcache_before):
    """The GPU's cosine scores of a layer against fp64 cosine of its own value vectors and the
    cached V rows the layer read."""
    n = cfg.gen_len
    N = cfg.seq_len
    sims = eng.buffer("scores")[:cfg.batch * n].double().cpu().numpy()
    vnew = eng.buffer("vnew")[:cfg.batch * n].double().cpu().numpy()
    flat = np.concatenate([b * N + cfg.prompt_len + np.arange(n) for b in range(cfg.batch)])
    vc = vcache_before.double().cpu().numpy()             # [B, Hkv, N, hd]
    vrows = vc[flat // N, :, flat % N, :].reshape(len(flat), -1)
    np.testing.assert_allclose(sims, cosine_rows(vnew, vrows), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("forced", [False, True])
def test_dllm_cache_capped_selection_teacher_forced(tiny_w, forced):
    """dLLM-Cache with tau = 0.95 and rho = 0.25: the oracle's per-layer similarities are fed to
    the GPU's selection (dllm_set_forced_similarities), and the rows chosen at every layer equal
    the oracle's, bit for bit; outputs agree within tolerance and the GPU's own cosine equals
    fp64 cosine of its own value vectors.  forced=True uses similarities where both the
    threshold and the cap bind (12 of 32 rows below 0.5, cap 8)."""
    cfg = TINY.replace(policy="dllm_cache", sim_tau=0.5 if forced else 0.95, rho_cap=0.25,
                       prompt_interval=5, tokens_per_step=2, batch=2)
    N, L, n = cfg.seq_len, cfg.model.n_layers, cfg.gen_len
    tok0 = make_tokens(cfg)
    orc = OracleRun(cfg, tiny_w, tok0.numpy())
    eng = Engine(cfg, _dev(tiny_w), tok0.to(DEV).contiguous())
    fsims = torch.zeros((L, cfg.batch, n), dtype=torch.float32, device=DEV)
    eng.set_forced_similarities(fsims)
    cap = math.ceil(cfg.rho_cap * n - 1e-9)
    rng = np.random.default_rng(5)
    n_partial = n_capped = 0
    while not orc.done:
        fs = None
        if forced and orc.n_steps % cfg.prompt_interval:
            fs = []
            for l in range(L):
                sims = np.full(cfg.batch * n, 0.9)
                for b in range(cfg.batch):
                    low = rng.choice(n, 12, replace=False)
                    sims[b * n + low] = rng.permutation(np.linspace(0.05, 0.45, 12))
                fs.append(sims)
        rec = orc.step(forced_scores=fs)
        kind = eng.begin_step()
        assert kind == ("full" if rec["kind"] == "refresh" else "partial")
        if kind == "partial":
            fsims.copy_(torch.tensor(np.stack([lay["sims"] for lay in rec["layers"]]).reshape(L, cfg.batch, n)))
        for l in range(L):
            vc0 = eng.buffer("vcache")[l].clone()
            eng.layer_forward(l)
            if kind == "partial":
                want = rec["layers"][l]["sel"]
                nsel = int(eng.buffer("nsel")[0])
                got = eng.buffer("selrows")[:nsel].cpu().numpy()
                np.testing.assert_array_equal(got, (want // n) * N + cfg.prompt_len + want % n)
                for b in range(cfg.batch):
                    sims_b = rec["layers"][l]["sims"][b * n:(b + 1) * n]
                    np.testing.assert_array_equal(
                        np.sort(want[(want >= b * n) & (want < (b + 1) * n)] - b * n),
                        threshold_cap_select(sims_b, cfg.sim_tau, cap))
                    n_capped += int((np.asarray(sims_b) < cfg.sim_tau).sum() > cap)
                _check_cos_on_own_values(eng, cfg, vc0)
        eng.unmask()
        torch.cuda.synchronize()
        b_idx, pos = rec["rows"]
        got = eng.buffer("hcache")[L - 1][torch.tensor(b_idx * N + pos, device=DEV)].cpu().numpy()
        assert _rowrel(got, rec["h_out"]) < TOL_HIDDEN
        n_partial += kind == "partial"
        _force(eng, orc)
    assert n_partial > 0 and eng.done
    if forced:
        assert n_capped > 0


def test_dllm_cache_dus_generation(tiny_w):
    cfg = TINY.replace(policy="dllm_cache", unmask="dus", block_len=8, prompt_interval=5,
                       sim_tau=0.95, rho_cap=0.25)
    N = cfg.seq_len
    eng = Engine(cfg, _dev(tiny_w), make_tokens(cfg).to(DEV).contiguous())
    rounds = dus_schedule(cfg.block_len)
    pos = torch.full((1, cfg.block_len), -1, dtype=torch.int32, device=DEV)
    tk = torch.full_like(pos, -1)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    steps, seen = 0, np.zeros(N, int)
    cap = math.ceil(cfg.rho_cap * cfg.gen_len)
    while not eng.done:
        block, r = divmod(steps, len(rounds))
        kind = eng.begin_step()
        for l in range(cfg.model.n_layers):
            eng.layer_forward(l)
            if kind == "partial":
                assert int(eng.buffer("nsel")[0]) <= cap
        eng.unmask(pos, tk, cnt)
        committed = sorted(pos[0, :int(cnt[0])].tolist())
        expect = sorted((cfg.prompt_len + block * cfg.block_len + rounds[r]).tolist())
        assert committed == expect                           # exactly this round's dilated group
        for p in committed:
            seen[p] += 1
        steps += 1
    assert steps == (cfg.gen_len // cfg.block_len) * len(rounds)
    assert np.all(seen[cfg.prompt_len:] == 1) and np.all(seen[:cfg.prompt_len] == 0)
    assert not bool((eng.tokens == cfg.model.mask_id).any())


def test_dllm_cache_forced_ratio_selects_exactly_the_cap(tiny_w):
    cfg = TINY.replace(policy="dllm_cache", unmask="dus", block_len=8, prompt_interval=100, rho_cap=0.25)
    eng = Engine(cfg, _dev(tiny_w), make_tokens(cfg).to(DEV).contiguous(), forced_rho=1)
    eng.step()                                               # refresh
    eng.begin_step()
    for l in range(cfg.model.n_layers):
        eng.layer_forward(l)
        assert int(eng.buffer("nsel")[0]) == math.ceil(0.25 * cfg.gen_len)
    eng.unmask()


# ------------------------------------------------------------------ confidence-bounded DUS

def test_cb_dus_generation(tiny_w):
    """The engine with confidence-bounded, dilation-filtered unmasking: every masked position is
    unmasked once, no two in one step are adjacent, at most tokens_per_step per step, and the
    data-dependent block ends are followed (the run takes fewer steps than one token per step)."""
    cfg = TINY.replace(policy="vanilla", unmask="cb_dus", cb_tau=0.0, tokens_per_step=4)
    eng = Engine(cfg, _dev(tiny_w), make_tokens(cfg).to(DEV).contiguous())
    pos = torch.full((1, 4), -1, dtype=torch.int32, device=DEV)
    tk = torch.full_like(pos, -1)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    seen = np.zeros(cfg.seq_len, int)
    steps = 0
    while not eng.done:
        eng.begin_step()
        for l in range(cfg.model.n_layers):
            eng.layer_forward(l)
        eng.unmask(pos, tk, cnt)
        ps = sorted(pos[0, :int(cnt[0])].tolist())
        assert 1 <= len(ps) <= 4 and all(q - p >= 2 for p, q in zip(ps, ps[1:]))
        for p in ps:
            seen[p] += 1
        steps += 1
    assert np.all(seen[cfg.prompt_len:] == 1) and np.all(seen[:cfg.prompt_len] == 0)
    assert steps < cfg.gen_len
    assert not bool((eng.tokens == cfg.model.mask_id).any())


def test_cb_dus_unreachable_bound_is_top1(tiny_w):
    """A bound no confidence reaches leaves the forced best token only: the same tokens as
    top-1 decoding (both on the kernel-per-step layer, whose sums are bit-reproducible; the
    fused layer adds fp32 pieces in arbitrary order)."""
    w = _dev(tiny_w)
    tok0 = make_tokens(TINY).to(DEV).contiguous()
    a = Engine(TINY.replace(policy="vanilla", unmask="cb_dus", cb_tau=2.0, tokens_per_step=4), w, tok0.clone(),
               layer_kernel="split")
    b = Engine(TINY.replace(policy="vanilla", unmask="topconf", tokens_per_step=1), w, tok0.clone(),
               layer_kernel="split")
    na = nb = 0
    while not a.done:
        a.step()
        na += 1
    while not b.done:
        b.step()
        nb += 1
    assert na == nb == TINY.gen_len
    assert torch.equal(a.tokens, b.tokens)

"""Per-kernel parity of the CUDA path against the oracle, through the C ABI.

Inputs are seeded and bf16-exact where the kernel reads bf16, so both sides
see the same numbers; the oracle computes in fp64.  Index outputs (selection,
unmasking) are compared bit for bit when both sides get the same scores.
Floating tolerances follow from the arithmetic: fp32 accumulation of exact
bf16 products (GEMM ~1e-5 relative) plus one bf16 rounding of each stored
activation (2^-8 relative).
"""
import math

import numpy as np
import pytest
import torch

from oracle import model as om
from oracle import policy as op
from synth.configs import ModelDims

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from token_skip_denoising_b200 import ops
    from token_skip_denoising_b200.engine import device_status

DEV = "cuda"


def _gen(seed):
    return torch.Generator(device="cpu").manual_seed(seed)


def _bf16(shape, seed, std=1.0):
    return (torch.randn(shape, generator=_gen(seed)) * std).to(torch.bfloat16)


def _f64(t):
    return t.detach().cpu().double().numpy()


def _rowrel(a, b):
    """max over rows of max|a - b| / max|b| (b is the reference)."""
    a = np.asarray(a, dtype=np.float64).reshape(len(a), -1)
    b = np.asarray(b, dtype=np.float64).reshape(len(b), -1)
    den = np.maximum(np.abs(b).max(axis=1), 1e-30)
    return float((np.abs(a - b).max(axis=1) / den).max())


# ------------------------------------------------------------------ GEMM

@pytest.mark.parametrize("rows,count,n_out,K,splits,bn", [
    (7, None, 384, 512, 0, 0), (16, None, 256, 256, 1, 0), (33, 29, 512, 1024, 3, 0),
    (100, None, 384, 512, 0, 0), (300, 257, 256, 512, 1, 0), (5, None, 128, 4096, 9, 0),
    (64, 50, 256, 512, 2, 128), (200, None, 128, 192, 0, 256),
    (600, 577, 256, 512, 0, 0), (520, None, 384, 1024, 0, 0),
])
def test_gemm_store_f32(rows, count, n_out, K, splits, bn):
    W = _bf16((n_out, K), 1, 0.05)
    X = _bf16((rows, K), 2)
    cnt = None if count is None else torch.tensor([count], dtype=torch.int32, device=DEV)
    out = torch.full((rows, n_out), 7.0, device=DEV)
    ops.gemm(W.to(DEV), X.to(DEV), kind=0, count=cnt, out=out, splits=splits, bn=bn)
    m = rows if count is None else count
    ref = _f64(X[:m]) @ _f64(W).T
    got = out.cpu().double().numpy()
    assert _rowrel(got[:m], ref) < 1e-4
    if m < rows:
        assert torch.all(out[m:] == 7.0)          # rows beyond the device count untouched


@pytest.mark.parametrize("splits", [1, 4])
def test_gemm_residual_scatter(splits):
    n_out, K, rows = 256, 1024, 9
    W = _bf16((n_out, K), 3, 0.05)
    X = _bf16((rows, K), 4)
    h0 = torch.randn((40, n_out), generator=_gen(5))
    rmap = torch.tensor([3, 5, 6, 10, 11, 20, 21, 33, 39], dtype=torch.int32)
    h = h0.clone().to(DEV)
    ops.gemm(W.to(DEV), X.to(DEV), kind=3, out=h, rows_map=rmap.to(DEV), splits=splits)
    ref = _f64(h0)
    ref[rmap.numpy()] += _f64(X) @ _f64(W).T
    got = h.cpu().double().numpy()
    assert _rowrel(got, ref) < 1e-5
    untouched = np.setdiff1d(np.arange(40), rmap.numpy())
    np.testing.assert_array_equal(got[untouched], _f64(h0)[untouched])


@pytest.mark.parametrize("rows,n_out,K,count", [(100, 1024, 2048, None), (205, 1024, 4096, 190), (768, 4096, 1024, None)])
def test_gemm_residual_wide_tiles(rows, n_out, K, count):
    """The residual add from 128-wide tiles on: at 100 and 205 rows (8 and 16 tiles, at most half
    the SMs) each piece of a split tile adds its own partial into h; at 768 rows with 4096 outputs
    the 128-wide tiles would outnumber the SMs, so it runs as 96 whole 256-wide tiles."""
    W = _bf16((n_out, K), 12, 0.05)
    X = _bf16((rows, K), 13)
    g = _gen(14)
    n_h = rows + 37
    h0 = torch.randn((n_h, n_out), generator=g)
    rmap = torch.randperm(n_h, generator=g)[:rows].to(torch.int32)
    cnt = None if count is None else torch.tensor([count], dtype=torch.int32, device=DEV)
    h = h0.clone().to(DEV)
    ops.gemm(W.to(DEV), X.to(DEV), kind=3, count=cnt, out=h, rows_map=rmap.to(DEV))
    m = rows if count is None else count
    ref = _f64(h0)
    ref[rmap[:m].numpy()] += _f64(X[:m]) @ _f64(W).T
    got = h.cpu().double().numpy()
    assert _rowrel(got, ref) < 1e-5
    untouched = np.setdiff1d(np.arange(n_h), rmap[:m].numpy())
    np.testing.assert_array_equal(got[untouched], _f64(h0)[untouched])


def test_gemm_split_k_is_deterministic():
    W = _bf16((512, 4096), 6, 0.05).to(DEV)
    X = _bf16((11, 4096), 7).to(DEV)
    a = ops.gemm(W, X, splits=8)
    b = ops.gemm(W, X, splits=8)
    assert torch.equal(a, b)


# ------------------------------------------------------------------ RMSNorm / embed

def test_rmsnorm_rows_gather():
    d = 512
    h = torch.randn((50, d), generator=_gen(8)) * 3
    g = 1 + 0.1 * torch.randn(d, generator=_gen(9))
    rows = torch.tensor([4, 0, 49, 17, 17, 8, 30], dtype=torch.int32)
    z = ops.rmsnorm_rows(h.to(DEV), g.to(DEV), 1e-5, rows=rows.to(DEV))
    ref = om.rmsnorm(_f64(h)[rows.numpy()], _f64(g), 1e-5)
    assert _rowrel(z.float().cpu().numpy(), ref) < 2 ** -8


def test_embed_rows():
    E = _bf16((64, 256), 10, 0.02)
    tokens = torch.randint(0, 64, (2, 40), generator=_gen(11), dtype=torch.int32)
    rows = torch.tensor([0, 5, 39, 40, 79], dtype=torch.int32)
    h = torch.full((80, 256), -1.0, device=DEV)
    ops.embed_rows(E.to(DEV), tokens.to(DEV), rows.to(DEV), None, 5, h)
    flat = tokens.reshape(-1)
    for r in rows.tolist():
        assert torch.equal(h[r].cpu(), E[flat[r]].float())
    assert torch.all(h[1] == -1.0)


def test_embed_rows_rejects_token_ids_outside_the_vocabulary():
    """The gather checks every id against the vocabulary before reading: an id outside it
    zeroes its row and sets DLLM_DEV_BAD_INDEX instead of reading past the table."""
    E = _bf16((64, 256), 10, 0.02)
    tokens = torch.tensor([[3, -1, 64, 2**31 - 1, 63]], dtype=torch.int32)
    rows = torch.arange(5, dtype=torch.int32)
    h = torch.full((5, 256), -1.0, device=DEV)
    assert device_status() == 0
    ops.embed_rows(E.to(DEV), tokens.to(DEV), rows.to(DEV), None, 5, h)
    assert device_status() == 2                     # DLLM_DEV_BAD_INDEX, and cleared
    assert torch.equal(h[0].cpu(), E[3].float()) and torch.equal(h[4].cpu(), E[63].float())
    assert torch.all(h[1:4] == 0.0)


# ------------------------------------------------------------------ QKV + RoPE, SwiGLU

@pytest.mark.parametrize("hq,hkv,hd,rows,splits", [(4, 4, 64, 9, 0), (8, 2, 128, 37, 1), (28, 4, 128, 5, 3),
                                                   (8, 2, 128, 100, 0), (28, 4, 128, 180, 0),
                                                   (8, 2, 128, 600, 0)])
def test_qkv_rope_and_cache_scatter(hq, hkv, hd, rows, splits):
    d = 512 if hq * hd <= 1024 else 3584
    dims = ModelDims(n_layers=1, d_model=d, n_heads=hq, n_kv_heads=hkv, head_dim=hd, ffn_dim=256, vocab=256,
                     mask_id=255, rope_theta=10000.0)
    B, N = 2, max(96, rows)
    W = _bf16((dims.qkv_dim, d), 12, 0.03)
    X = _bf16((rows, d), 13)
    rng = np.random.default_rng(14)
    flat = np.sort(rng.choice(B * N, rows, replace=False)).astype(np.int32)
    cos, sin = ops.rope_table(N, hd, dims.rope_theta)
    kc = torch.zeros((B, hkv, N, hd), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    q = ops.qkv_rope(W.to(DEV), X.to(DEV), dims, N, torch.tensor(flat, device=DEV), cos, sin, kc, vc, splits=splits)
    y = _f64(X) @ _f64(W).T
    pos = flat % N
    qr = om.apply_rope(y[:, :dims.q_dim].reshape(rows, hq, hd), pos, dims.rope_theta)
    kr = om.apply_rope(y[:, dims.q_dim:dims.q_dim + dims.kv_dim].reshape(rows, hkv, hd), pos, dims.rope_theta)
    vr = y[:, dims.q_dim + dims.kv_dim:].reshape(rows, hkv, hd)
    assert _rowrel(q.float().cpu().numpy(), qr.reshape(rows, -1)) < 1e-2
    kg = kc.float().cpu().numpy()
    vg = vc.float().cpu().numpy()
    for j, f in enumerate(flat):
        b, p = divmod(int(f), N)
        assert _rowrel(kg[b, :, p].reshape(1, -1), kr[j].reshape(1, -1)) < 1e-2
        assert _rowrel(vg[b, :, p].reshape(1, -1), vr[j].reshape(1, -1)) < 1e-2
    # rows not in the map stay zero
    written = np.zeros(B * N, bool)
    written[flat] = True
    for f in np.nonzero(~written)[0][:10]:
        b, p = divmod(int(f), N)
        assert np.all(kg[b, :, p] == 0)


def test_qkv_rope_beyond_the_grid_height():
    """70000 rows: the RoPE pass covers rows past the 65535-row grid height by striding."""
    hq, hkv, hd, d, rows = 2, 2, 64, 64, 70000
    dims = ModelDims(n_layers=1, d_model=d, n_heads=hq, n_kv_heads=hkv, head_dim=hd, ffn_dim=256, vocab=256,
                     mask_id=255, rope_theta=10000.0)
    N = rows
    W = _bf16((dims.qkv_dim, d), 15, 0.1)
    X = _bf16((rows, d), 16)
    flat = np.random.default_rng(17).permutation(N).astype(np.int32)
    cos, sin = ops.rope_table(N, hd, dims.rope_theta)
    kc = torch.zeros((1, hkv, N, hd), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    ws = torch.zeros(512 << 20, dtype=torch.uint8, device=DEV)
    q = ops.qkv_rope(W.to(DEV), X.to(DEV), dims, N, torch.tensor(flat, device=DEV), cos, sin, kc, vc, ws=ws)
    torch.cuda.synchronize()
    y = _f64(X) @ _f64(W).T
    qr = om.apply_rope(y[:, :dims.q_dim].reshape(rows, hq, hd), flat, dims.rope_theta)
    kr = om.apply_rope(y[:, dims.q_dim:dims.q_dim + dims.kv_dim].reshape(rows, hkv, hd), flat, dims.rope_theta)
    assert _rowrel(q.float().cpu().numpy(), qr.reshape(rows, -1)) < 1e-2
    kg = kc[0].float().cpu().numpy().transpose(1, 0, 2)[flat]          # [rows, hkv, hd] in row order
    vg = vc[0].float().cpu().numpy().transpose(1, 0, 2)[flat]
    assert _rowrel(kg.reshape(rows, -1), kr.reshape(rows, -1)) < 1e-2
    assert _rowrel(vg.reshape(rows, -1), y[:, dims.q_dim + dims.kv_dim:]) < 1e-2


@pytest.mark.parametrize("rows,F,splits", [(3, 256, 0), (40, 1024, 1), (130, 512, 0), (8, 18944 // 4, 2),
                                           (400, 512, 0), (700, 256, 0)])
def test_gate_up_swiglu(rows, F, splits):
    d = 512
    W = _bf16((2 * F, d), 15, 0.04)
    X = _bf16((rows, d), 16)
    act = ops.gate_up(W.to(DEV), X.to(DEV), F, splits=splits)
    gu = _f64(X) @ _f64(W).T
    ref = om.silu(gu[:, :F]) * gu[:, F:]
    assert _rowrel(act.float().cpu().numpy(), ref) < 1e-2


# ------------------------------------------------------------------ attention

@pytest.mark.parametrize("B,counts,N,hq,hkv,hd,splits", [
    (1, [7], 768, 4, 4, 128, 0), (1, [7], 768, 4, 4, 128, 1), (2, [3, 70], 100, 4, 2, 128, 0),
    (1, [130], 130, 2, 2, 64, 3), (3, [1, 0, 17], 64, 7, 1, 128, 2), (1, [32], 2048, 2, 2, 128, 0),
])
def test_attention_vs_oracle(B, counts, N, hq, hkv, hd, splits):
    dims = ModelDims(n_layers=1, d_model=hq * hd, n_heads=hq, n_kv_heads=hkv, head_dim=hd, ffn_dim=64, vocab=128,
                     mask_id=127)
    rows = sum(counts)
    q = _bf16((max(rows, 1), hq * hd), 20)
    K = _bf16((B, hkv, N, hd), 21)
    V = _bf16((B, hkv, N, hd), 22)
    off = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32)
    out = ops.attention(q.to(DEV), K.to(DEV), V.to(DEV), off.to(DEV), dims, max(counts), splits=splits)
    got = out.float().cpu().numpy()
    qd = _f64(q).reshape(-1, hq, hd)
    for b in range(B):
        s, e = int(off[b]), int(off[b + 1])
        if e == s:
            continue
        ref = om.attention(qd[s:e], _f64(K[b]), _f64(V[b])).reshape(e - s, -1)
        assert _rowrel(got[s:e], ref) < 2e-2


# Tensor-core path (head dim 128, >= 64 query units per sequence and KV head): the refresh
# shape (every row of the sequence), a Dream-7B GQA group (7 query heads per KV head), a
# ragged last key tile, forced key splits and sequences of unequal length.  The operands are
# bf16 on both sides, so what remains is the bf16 rounding of P (2^-9 of the largest weight)
# and of the output: 8e-3 of each row's largest entry.
TOL_ATTN_TC = 8e-3


@pytest.mark.parametrize("B,counts,N,hq,hkv,splits", [
    (1, [768], 768, 4, 4, 0), (1, [300], 1536, 28, 4, 0), (1, [200], 1000, 2, 2, 3),
    (2, [129, 64], 300, 4, 4, 0), (2, [70, 5], 2048, 2, 2, 0), (1, [64], 128, 1, 1, 1),
])
def test_attention_tensor_core_vs_oracle(B, counts, N, hq, hkv, splits):
    hd = 128
    dims = ModelDims(n_layers=1, d_model=hq * hd, n_heads=hq, n_kv_heads=hkv, head_dim=hd, ffn_dim=64, vocab=128,
                     mask_id=127)
    rows = sum(counts)
    q = _bf16((rows, hq * hd), 30)
    K = _bf16((B, hkv, N, hd), 31)
    V = _bf16((B, hkv, N, hd), 32)
    off = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32)
    out = ops.attention(q.to(DEV), K.to(DEV), V.to(DEV), off.to(DEV), dims, max(counts), splits=splits)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    qd = _f64(q).reshape(-1, hq, hd)
    for b in range(B):
        s, e = int(off[b]), int(off[b + 1])
        ref = om.attention(qd[s:e], _f64(K[b]), _f64(V[b])).reshape(e - s, -1)
        err = _rowrel(got[s:e], ref)
        assert err < TOL_ATTN_TC, (b, err)


@pytest.mark.parametrize("ramp", [0.05, -0.05])
def test_attention_tensor_core_rescale(ramp):
    """Scores that climb (or fall) along the keys: every query shares a direction d with
    |d|^2 = 16 and key n carries n * ramp * d, so S' moves by ~13 per 128-key tile.  Climbing,
    each tile's maximum exceeds the running offset by more than the slack and O, l are
    rescaled at every tile; falling, the first tile holds the maximum and nothing is."""
    hd, hq, hkv, N, rows = 128, 2, 2, 1000, 200
    dims = ModelDims(n_layers=1, d_model=hq * hd, n_heads=hq, n_kv_heads=hkv, head_dim=hd, ffn_dim=64, vocab=128,
                     mask_id=127)
    g = torch.Generator().manual_seed(40)
    d = torch.zeros(hd)
    d[:16] = 1.0
    q = (torch.randn((rows, hq, hd), generator=g) * 0.3 + d).reshape(rows, hq * hd).to(torch.bfloat16)
    pos = torch.arange(N, dtype=torch.float32)[:, None]
    K = (torch.randn((1, hkv, N, hd), generator=g) * 0.3 + (pos * ramp) * d).to(torch.bfloat16)
    V = _bf16((1, hkv, N, hd), 41)
    off = torch.tensor([0, rows], dtype=torch.int32)
    out = ops.attention(q.to(DEV), K.to(DEV), V.to(DEV), off.to(DEV), dims, rows)
    torch.cuda.synchronize()
    ref = om.attention(_f64(q).reshape(rows, hq, hd), _f64(K[0]), _f64(V[0])).reshape(rows, -1)
    assert _rowrel(out.float().cpu().numpy(), ref) < TOL_ATTN_TC


# ------------------------------------------------------------------ LM head

@pytest.mark.parametrize("rows,V,count", [(7, 1024, None), (32, 4096, 20), (3, 126464 // 4, None)])
def test_lm_head_confidence(rows, V, count):
    d = 512
    W = _bf16((V, d), 23, 0.05)
    X = _bf16((rows, d), 24)
    mask_id = V - 1
    cnt = None if count is None else torch.tensor([count], dtype=torch.int32, device=DEV)
    conf, amax, lse = ops.lm_head(W.to(DEV), X.to(DEV), mask_id, count=cnt)
    m = rows if count is None else count
    z = _f64(X[:m]) @ _f64(W).T
    rc, rt, rl = om.lm_confidence(z, mask_id)
    gc, gt, gl = conf[:m].cpu().numpy(), amax[:m].cpu().numpy(), lse[:m].cpu().numpy()
    np.testing.assert_allclose(gl, rl, rtol=1e-5, atol=1e-4)
    for j in range(m):
        assert gt[j] != mask_id
        # the chosen token is a maximiser of the exact logits up to fp32 accumulation error
        assert z[j, gt[j]] >= z[j, rt[j]] - 1e-4 * max(1.0, abs(z[j, rt[j]]))
        assert abs(gc[j] - math.exp(z[j, gt[j]] - rl[j])) <= 1e-4 * gc[j] + 1e-7


def test_lm_head_excludes_mask_id():
    d, V = 256, 256
    W = _bf16((V, d), 25, 0.05)
    X = _bf16((4, d), 26)
    z = _f64(X) @ _f64(W).T
    mask_id = int(np.argmax(z[0]))                # the mask id holds row 0's largest logit
    conf, amax, lse = ops.lm_head(W.to(DEV), X.to(DEV), mask_id)
    assert int(amax[0]) != mask_id
    _, rt, _ = om.lm_confidence(z, mask_id)
    assert int(amax[0]) == int(rt[0])


# ------------------------------------------------------------------ scores

def test_score_es_matches_eq1():
    n, d = 37, 4096
    h = torch.randn((n, d), generator=_gen(30))
    hp = torch.randn((n, d), generator=_gen(31))
    hp[5] = 0.0                                       # zero previous state -> variation 0
    conf = torch.rand(n, generator=_gen(32))
    mp = (torch.rand(n, generator=_gen(33)) < 0.5).to(torch.uint8)
    s = ops.score_es(h.to(DEV), hp.to(DEV), conf.to(DEV), 0.5, masked_prev=mp.to(DEV))
    c = np.where(mp.numpy() > 0, _f64(conf), 0.0)
    ref = op.es_importance(0.5, c, _f64(h), _f64(hp))
    np.testing.assert_allclose(s.cpu().numpy(), ref, rtol=2e-5, atol=1e-7)


def test_score_es_update_rolls_state():
    n, d, mask = 8, 256, 99
    h = torch.randn((n, d), generator=_gen(34)).to(DEV)
    hp = torch.randn((n, d), generator=_gen(35)).to(DEV)
    conf = torch.rand(n, generator=_gen(36)).to(DEV)
    mp = torch.ones(n, dtype=torch.uint8, device=DEV)
    tok = torch.tensor([99, 1, 99, 2, 3, 99, 4, 5], dtype=torch.int32, device=DEV)
    rows = torch.tensor([1, 3, 6], dtype=torch.int32, device=DEV)
    hp0 = hp.clone()
    ops.score_es(h, hp, conf, 0.3, rows=rows, masked_prev=mp, tokens=tok, mask_id=mask, update=1)
    for r in range(n):
        if r in (1, 3, 6):
            assert torch.equal(hp[r], h[r]) and int(mp[r]) == 0
        else:
            assert torch.equal(hp[r], hp0[r]) and int(mp[r]) == 1


def test_score_cos_matches_oracle():
    B, N, hkv, hd = 2, 50, 4, 128
    vc = _bf16((B, hkv, N, hd), 37)
    rows = torch.tensor([0, 7, 49, 50, 99, 60], dtype=torch.int32)
    vnew = torch.randn((6, hkv * hd), generator=_gen(38))
    vnew[2] = 0.0
    vc[1, :, 10] = 0.0                       # flat 60 -> (1, 10): cached zero, new nonzero
    s = ops.score_cos(vnew.to(DEV), vc.to(DEV), rows.to(DEV), N, hkv, hd)
    vcf = _f64(vc)
    ref_c = np.stack([vcf[f // N, :, f % N].reshape(-1) for f in rows.tolist()])
    ref = op.cosine_rows(_f64(vnew), ref_c)
    np.testing.assert_allclose(s.cpu().numpy(), ref, rtol=1e-5, atol=1e-6)
    assert float(s[2]) == 0.0 and float(s[5]) == 0.0


def test_kl_conf_matches_oracle():
    rows, V = 6, 5000
    z = _bf16((rows, V), 39, 2.0)
    zp = _bf16((rows, V), 40, 2.0)
    zp[1] = z[1]                                       # identical distribution -> KL 0
    zpf, zf = _f64(zp), _f64(z)
    lse_p = torch.tensor([float(np.log(np.exp(r - r.max()).sum()) + r.max()) for r in zpf], dtype=torch.float32)
    has = torch.tensor([1, 1, 0, 1, 1, 1], dtype=torch.int32)
    rows_idx = torch.arange(rows, dtype=torch.int32)
    conf, amax, lse, kl = ops.kl_conf(z.to(DEV), V - 1, rows=rows_idx.to(DEV), zp_store=zp.to(DEV),
                                      lse_prev=lse_p.to(DEV), has_prev=has.to(DEV))
    rc, rt, rl = om.lm_confidence(zf, V - 1)
    np.testing.assert_allclose(lse.cpu().numpy(), rl, rtol=1e-6, atol=1e-5)
    np.testing.assert_array_equal(amax.cpu().numpy(), rt)      # bf16 logits: exact maxima
    np.testing.assert_allclose(conf.cpu().numpy(), rc, rtol=1e-4)
    ref_kl = op.kl_from_logits(zf, rl, zpf, _f64(lse_p))
    g = kl.cpu().numpy()
    assert math.isnan(g[2])
    ok = np.array([0, 1, 3, 4, 5])
    np.testing.assert_allclose(g[ok], ref_kl[ok], rtol=1e-3, atol=2e-5)
    assert abs(g[1]) < 2e-5 and np.all(g[ok] >= 0)


def test_kl_conf_large_vocab_and_shape_guard():
    """The one-pass statistics at the Dream-7B vocabulary (152064 = 8 x 19008, several thousand
    16-byte loads per thread) against fp64, and a vocabulary that is not a multiple of 8 refused
    (the kernel reads rows in 16-byte vectors)."""
    rows, V = 3, 152064
    z = _bf16((rows, V), 41, 3.0)
    zp = _bf16((rows, V), 42, 3.0)
    zf, zpf = _f64(z), _f64(zp)
    lse_p = torch.tensor([float(np.log(np.exp(r - r.max()).sum()) + r.max()) for r in zpf], dtype=torch.float32)
    has = torch.ones(rows, dtype=torch.int32)
    conf, amax, lse, kl = ops.kl_conf(z.to(DEV), V - 1, rows=torch.arange(rows, dtype=torch.int32).to(DEV),
                                      zp_store=zp.to(DEV), lse_prev=lse_p.to(DEV), has_prev=has.to(DEV))
    rc, rt, rl = om.lm_confidence(zf, V - 1)
    np.testing.assert_allclose(lse.cpu().numpy(), rl, rtol=1e-6, atol=1e-5)
    np.testing.assert_array_equal(amax.cpu().numpy(), rt)
    np.testing.assert_allclose(conf.cpu().numpy(), rc, rtol=1e-4)
    np.testing.assert_allclose(kl.cpu().numpy(), op.kl_from_logits(zf, rl, zpf, _f64(lse_p)), rtol=1e-3, atol=2e-5)
    from token_skip_denoising_b200._lib import DllmError
    with pytest.raises(DllmError):
        ops.kl_conf(_bf16((2, 1001), 43).to(DEV), 1000)


# ------------------------------------------------------------------ selection (bit-exact)

def _scores_with_ties(B, n, seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(0, 6, (B, n)).astype(np.float32) / 5
    s += (rng.random((B, n)) < 0.3) * rng.random((B, n)).astype(np.float32)
    return s.astype(np.float32)


@pytest.mark.parametrize("B,n,k", [(1, 32, 7), (1, 32, 8), (3, 1024, 256), (2, 2048, 62), (1, 5, 5),
                                   (4, 1536, 1), (1, 3000, 2999), (2, 64, 0)])
def test_select_topk_bit_exact(B, n, k):
    s = _scores_with_ties(B, n, n + k)
    act, cnt, rows, off = ops.select(torch.tensor(s, device=DEV), B, n, ops.SEL_TOPK_DESC, k, cand_start=11, N=n + 20)
    for b in range(B):
        ref = op.topk_select(s[b].astype(np.float64), k) + 11
        kk = len(ref)
        assert int(cnt[b]) == kk
        np.testing.assert_array_equal(act[b, :kk].cpu().numpy(), ref)
        assert int(off[b]) == b * kk
        np.testing.assert_array_equal(rows[b * kk:(b + 1) * kk].cpu().numpy(), b * (n + 20) + ref)
    assert int(off[B]) == B * min(k, n)


def test_select_nan_and_negative_zero():
    s = np.array([[np.nan, -0.0, 0.0, -1.0, np.inf, -np.inf]], dtype=np.float32)
    for k in range(7):
        act, cnt, _, _ = ops.select(torch.tensor(s, device=DEV), 1, 6, ops.SEL_TOPK_DESC, k, k_max=6)
        ref = op.topk_select(s[0].astype(np.float64), k)
        assert int(cnt[0]) == len(ref)
        np.testing.assert_array_equal(act[0, :len(ref)].cpu().numpy(), ref)


@pytest.mark.parametrize("B,n,cap,tau,forced", [(4, 1024, 256, 0.95, False), (2, 100, 7, 0.5, False),
                                                 (1, 2048, 512, -5.0, True), (3, 40, 40, 2.0, False)])
def test_select_threshold_cap_bit_exact(B, n, cap, tau, forced):
    s = _scores_with_ties(B, n, 7 * n + cap)
    s[0, 3] = np.nan
    mode = ops.SEL_FORCED_ASC if forced else ops.SEL_BELOW_CAP_ASC
    act, cnt, rows, off = ops.select(torch.tensor(s, device=DEV), B, n, mode, cap, tau=tau, k_max=max(cap, 1))
    total = 0
    for b in range(B):
        ref = op.threshold_cap_select(s[b].astype(np.float64), tau, cap, forced=forced)
        kk = len(ref)
        assert int(cnt[b]) == kk
        np.testing.assert_array_equal(act[b, :kk].cpu().numpy(), ref)
        assert int(off[b]) == total
        total += kk
    assert int(off[B]) == total


def test_select_all_unlocked():
    B, N = 3, 200
    rng = np.random.default_rng(50)
    lock = (rng.random((B, N)) < 0.4).astype(np.uint8)
    act, cnt, rows, off = ops.select(None, B, N, ops.SEL_ALL_ELIGIBLE, 0, N=N, lock=torch.tensor(lock, device=DEV))
    total = 0
    for b in range(B):
        ref = np.nonzero(lock[b] == 0)[0]
        assert int(cnt[b]) == len(ref)
        np.testing.assert_array_equal(rows[total:total + len(ref)].cpu().numpy(), b * N + ref)
        total += len(ref)


# ------------------------------------------------------------------ unmasking (bit-exact)

@pytest.mark.parametrize("n_commit", [1, 4])
def test_unmask_topconf_bit_exact(n_commit):
    B, P, blk = 3, 16, 32
    N = P + 2 * blk
    rng = np.random.default_rng(60 + n_commit)
    mask = 999
    tok = np.full((B, N), mask, dtype=np.int32)
    tok[:, :P] = rng.integers(0, 900, (B, P))
    tok[:, P + 3] = 5                                   # already unmasked in block 0
    conf = (rng.integers(0, 8, (B, N)) / 8).astype(np.float32)
    amax = rng.integers(0, 900, (B, N)).astype(np.int32)
    t = torch.tensor(tok, device=DEV)
    pos, tk, cnt = ops.unmask(t, torch.tensor(conf.reshape(-1), device=DEV), torch.tensor(amax.reshape(-1), device=DEV),
                              P, blk, mask, n_commit)
    got = t.cpu().numpy()
    for b in range(B):
        masked = tok[b, P:P + blk] == mask
        ref = op.unmask_topconf(conf[b, P:P + blk].astype(np.float64), masked, n_commit) + P
        exp = tok[b].copy()
        exp[ref] = amax[b, ref]
        np.testing.assert_array_equal(got[b], exp)
        assert int(cnt[b]) == len(ref)
        assert sorted(pos[b, :len(ref)].tolist()) == ref.tolist()


@pytest.mark.parametrize("blk,tau,cap", [(32, 0.5, 4), (32, 2.0, 4), (200, 0.0, 64), (1000, 0.3, 7), (64, -1.0, 64)])
def test_unmask_cb_dus_bit_exact(blk, tau, cap):
    """Confidence-bounded, dilation-filtered unmasking against the oracle's rule, with ties
    (confidences on a coarse grid), already-unmasked positions, ragged block lengths; and the
    count of masked positions left in the block."""
    B, P = 3, 8
    N = P + blk + 5
    rng = np.random.default_rng(blk + cap)
    mask = 999
    tok = np.full((B, N), mask, dtype=np.int32)
    tok[:, :P] = rng.integers(0, 900, (B, P))
    tok[:, P:P + blk][rng.random((B, blk)) < 0.3] = 7                  # some already unmasked
    conf = (rng.integers(0, 16, (B, N)) / 16).astype(np.float32)
    conf[0, P + 1] = np.nan                                             # NaN ranks last
    amax = rng.integers(0, 900, (B, N)).astype(np.int32)
    t = torch.tensor(tok, device=DEV)
    remain = torch.full((B,), -1, dtype=torch.int32, device=DEV)
    pos, tk, cnt = ops.unmask(t, torch.tensor(conf.reshape(-1), device=DEV), torch.tensor(amax.reshape(-1), device=DEV),
                              P, blk, mask, cap, max_out=cap, mode=ops.UNMASK_CB_DUS, cb_tau=tau, remain=remain)
    got = t.cpu().numpy()
    for b in range(B):
        masked = tok[b, P:P + blk] == mask
        ref = op.unmask_cb_dus(conf[b, P:P + blk], masked, tau, cap) + P
        exp = tok[b].copy()
        exp[ref] = amax[b, ref]
        np.testing.assert_array_equal(got[b], exp)
        assert int(cnt[b]) == len(ref)
        assert sorted(pos[b, :len(ref)].tolist()) == ref.tolist()
        assert int(remain[b]) == int(masked.sum()) - len(ref)


def test_unmask_dus_round():
    B, P, blk = 2, 8, 64
    N = P + blk
    mask = 77
    tok = np.full((B, N), mask, dtype=np.int32)
    tok[:, :P] = 3
    rounds = op.dus_schedule(blk)
    rm = np.zeros(blk, np.uint8)
    rm[rounds[2]] = 1
    amax = np.arange(B * N, dtype=np.int32) % 50
    t = torch.tensor(tok, device=DEV)
    ops.unmask(t, torch.zeros(B * N, device=DEV), torch.tensor(amax, device=DEV), P, blk, mask, 1,
               round_mask=torch.tensor(rm, device=DEV))
    got = t.cpu().numpy()
    for b in range(B):
        exp = tok[b].copy()
        exp[P + rounds[2]] = amax.reshape(B, N)[b, P + rounds[2]]
        np.testing.assert_array_equal(got[b], exp)

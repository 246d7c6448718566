"""A layer checked kernel by kernel on the operands the GPU itself produced.

The bf16 path rounds every stored activation to bf16 (the GEMM operands, the
rotated queries, the K/V cache, the attention output, the SwiGLU output).
Against the fp64 oracle run from the layer's input those roundings compound,
which is why a hidden state is held to 2e-2.  A mistake smaller than that
(a dropped term, a slightly wrong scale) would hide under it.  So here every
kernel of the layer is compared with fp64 arithmetic applied to the bf16
operands the GPU handed it, which leaves only fp32 accumulation and the one
rounding of the kernel's own output:

* the residual stream (fp32): h_out = h_in + W_o attn + W_down act, from the
  GPU's bf16 attn and act, to 1e-4 (fp32 accumulation over K <= 18944 terms);
* the SwiGLU output and the rotated q (stored in bf16): to 4e-3, one bf16
  rounding (2^-9 of the largest entry) with room for the fp32 sums;
* the attention output from the GPU's own q and K/V cache: to 8e-3 (the bf16
  probabilities of the P V product add one more 2^-9 rounding).

Both layer kernels are covered: the persistent fused kernel (its FFN operand is
g * h with 1/rms applied to the sums) and the kernel-per-step layer at the
LLaDA-8B width over 768 rows and the Dream-7B GQA width over 1536 rows.  The
formulas are the textbook block of the oracle's backbone (pre-norm attention
and SwiGLU); RoPE rotates pairs (i, i + hd/2).
"""
import numpy as np
import pytest
import torch

from synth import get_config, make_tokens, make_weights
from synth.configs import DREAM7B, LLADA8B, ModelDims, RunConfig, scaled

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from token_skip_denoising_b200.engine import Engine, device_status

DEV = "cuda"
TOL_RESID = 1e-4
TOL_BF16_OUT = 4e-3
TOL_ATTN = 8e-3


def _rowrel(a, b):
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    return float((np.abs(a - b).max(1) / np.maximum(np.abs(b).max(1), 1e-30)).max())


def _t64(x):
    return x.detach().to("cpu", torch.float64)


def _rope(x, pos, theta):
    """x [m, H, hd] float64, pairs (i, i + hd/2) rotated by pos * theta^(-2i/hd)."""
    hd = x.shape[-1]
    half = hd // 2
    inv = theta ** (-2.0 * torch.arange(half, dtype=torch.float64) / hd)
    ang = pos.to(torch.float64)[:, None] * inv[None, :]
    c, s = torch.cos(ang)[:, None, :], torch.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)


def _attention(q, K, V):
    """q [m, Hq, hd]; K, V [Hkv, N, hd] (one sequence), float64 softmax(q k^T / sqrt(hd)) v."""
    hq, hkv, hd = q.shape[1], K.shape[0], q.shape[2]
    out = torch.empty_like(q)
    for j in range(hq):
        kv = (j * hkv) // hq
        s = (q[:, j, :] @ K[kv].T) / np.sqrt(hd)
        out[:, j, :] = torch.softmax(s, dim=-1) @ V[kv]
    return out


def _check_layer(eng, dims, layer, rows_flat, h_in, kc_before_rows, fused, N, tag):
    """Compare the layer just run on rows_flat (flat b * N + pos) with fp64 on its own operands."""
    m = dims
    w = eng.weights
    li = layer
    Wqkv = _t64(w["w_qkv"][li])
    Wo, Wgu, Wd = _t64(w["w_o"][li]), _t64(w["w_gu"][li]), _t64(w["w_down"][li])
    ga, gf = _t64(w["g_attn"][li]), _t64(w["g_ffn"][li])
    n = len(rows_flat)
    idx = torch.tensor(rows_flat, device=DEV)
    h_out = _t64(eng.buffer("hidden")[idx])
    q_gpu = _t64(eng.buffer("layer_q")[:n])
    attn_gpu = _t64(eng.buffer("layer_attn")[:n])
    act_gpu = _t64(eng.buffer("layer_act")[:n])
    z2_gpu = _t64(eng.buffer("layer_z")[:n])
    kc = eng.buffer("kcache")[li].to("cpu", torch.float64)
    vc = eng.buffer("vcache")[li].to("cpu", torch.float64)
    b_idx = torch.tensor(np.asarray(rows_flat) // N)
    pos = torch.tensor(np.asarray(rows_flat) % N)

    # residual stream: h_out = h_in + W_o attn + W_down act (fp32 accumulation on both GEMMs)
    want = h_in + attn_gpu @ Wo.T + act_gpu @ Wd.T
    assert _rowrel(h_out, want) < TOL_RESID, (tag, "residual", _rowrel(h_out, want))

    # SwiGLU on the FFN operand of h_mid = h_in + W_o attn
    h_mid = h_in + attn_gpu @ Wo.T
    F = m.ffn_dim
    if fused:   # operand g * h, the sums scaled by 1/rms of h_mid
        r = 1.0 / torch.sqrt((h_mid * h_mid).mean(1, keepdim=True) + m.rms_eps)
        gu = (z2_gpu @ Wgu.T) * r
    else:       # operand bf16(RMSNorm(h_mid) * g)
        gu = z2_gpu @ Wgu.T
    act = gu[:, :F] / (1.0 + torch.exp(-gu[:, :F])) * gu[:, F:]
    assert _rowrel(act_gpu, act) < TOL_BF16_OUT, (tag, "swiglu", _rowrel(act_gpu, act))

    # rotated q and the new K/V rows from the QKV operand of h_in
    if fused:
        z1 = (_t64(eng.weights["g_attn"][li]).float() * h_in.float()).to(torch.bfloat16).double()
        r1 = 1.0 / torch.sqrt((h_in * h_in).mean(1, keepdim=True) + m.rms_eps)
        y = (z1 @ Wqkv.T) * r1
    else:
        z1 = (h_in / torch.sqrt((h_in * h_in).mean(1, keepdim=True) + m.rms_eps) * ga).float().to(torch.bfloat16)
        y = z1.double() @ Wqkv.T
    qd, kvd, hd = m.q_dim, m.kv_dim, m.head_dim
    q = _rope(y[:, :qd].reshape(n, m.n_heads, hd), pos, m.rope_theta).reshape(n, qd)
    k = _rope(y[:, qd:qd + kvd].reshape(n, m.n_kv_heads, hd), pos, m.rope_theta)
    v = y[:, qd + kvd:].reshape(n, m.n_kv_heads, hd)
    assert _rowrel(q_gpu, q) < TOL_BF16_OUT, (tag, "q", _rowrel(q_gpu, q))
    k_gpu = kc[b_idx, :, pos, :]
    v_gpu = vc[b_idx, :, pos, :]
    assert _rowrel(k_gpu.reshape(n, -1), k.reshape(n, -1)) < TOL_BF16_OUT, (tag, "k")
    assert _rowrel(v_gpu.reshape(n, -1), v.reshape(n, -1)) < TOL_BF16_OUT, (tag, "v")
    # rows outside the set kept their cached K/V
    if kc_before_rows is not None:
        kb = kc_before_rows.to("cpu", torch.float64)
        mask = torch.ones(kb.shape[0], kb.shape[2], dtype=torch.bool)
        mask[b_idx, pos] = False
        bb, pp = torch.nonzero(mask, as_tuple=True)
        assert torch.equal(kc[bb, :, pp, :], kb[bb, :, pp, :]), (tag, "untouched K rows")

    # attention of the GPU's own q over the GPU's own (updated) cache, per sequence
    qh = q_gpu.reshape(n, m.n_heads, hd)
    att = torch.empty_like(qh)
    for b in torch.unique(b_idx).tolist():
        sel = torch.nonzero(b_idx == b, as_tuple=True)[0]
        att[sel] = _attention(qh[sel], kc[b], vc[b])
    assert _rowrel(attn_gpu, att.reshape(n, qd)) < TOL_ATTN, (tag, "attention", _rowrel(attn_gpu, att.reshape(n, qd)))


def _one_layer(dims):
    return ModelDims(n_layers=1, d_model=dims.d_model, n_heads=dims.n_heads, n_kv_heads=dims.n_kv_heads,
                     head_dim=dims.head_dim, ffn_dim=dims.ffn_dim, vocab=1024, mask_id=1023,
                     rope_theta=dims.rope_theta)


@pytest.mark.parametrize("layer_kernel", ["fused", "split"])
@pytest.mark.parametrize("batch", [1, 2])
def test_skip_step_layers_kernel_by_kernel(layer_kernel, batch):
    """Both layers of a tiny skip step (32 candidate rows, then the 8 kept rows)."""
    cfg = get_config("tiny").replace(batch=batch)
    w = make_weights(cfg.model, device=DEV, gain_jitter=0.1)
    eng = Engine(cfg, w, make_tokens(cfg).to(DEV).contiguous(), layer_kernel=layer_kernel)
    eng.step()                                   # refresh fills the caches
    assert eng.begin_step() == "skip"
    N = cfg.seq_len
    for layer in range(cfg.model.n_layers):
        if layer == cfg.skip_layer:
            eng.select_active()
        n = int(eng.buffer("nrows")[0])
        rows = eng.buffer("rows")[:n].cpu().numpy().copy()
        h_in = _t64(eng.buffer("hidden")[torch.tensor(rows, device=DEV)])
        kc0 = eng.buffer("kcache")[layer].clone()
        eng.layer_forward(layer)
        torch.cuda.synchronize()
        assert device_status() == 0
        _check_layer(eng, cfg.model, layer, rows, h_in, kc0, layer_kernel == "fused", N,
                     f"{layer_kernel} layer {layer}")


@pytest.mark.parametrize("dims,N,B", [(LLADA8B, 768, 1), (DREAM7B, 1536, 1), (scaled(get_config("tiny"),
                                      n_kv_heads=2).model, 192, 3)])
def test_refresh_layer_kernel_by_kernel(dims, N, B):
    """The refresh path (every row of the sequence through the kernel-per-step layer): the
    LLaDA-8B width over 768 rows (128-wide GEMM tiles, 768 x 768 attention), the Dream-7B GQA
    width over 1536 rows (256-wide tiles), a GQA toy with 3 sequences."""
    d1 = _one_layer(dims)
    run = RunConfig(name="t", model=d1, batch=B, prompt_len=N - 64, gen_len=64, block_len=32,
                    policy="vanilla")
    w = make_weights(d1, device=DEV, gain_jitter=0.1, std=0.02)
    eng = Engine(run, w, make_tokens(run).to(DEV).contiguous())
    assert eng.begin_step() == "full"
    rows = np.arange(B * N)
    h_in = _t64(eng.buffer("hidden")[:B * N])
    eng.layer_forward(0)
    torch.cuda.synchronize()
    assert device_status() == 0
    _check_layer(eng, d1, 0, rows, h_in, None, False, N, f"refresh {d1.d_model}x{N}")

"""A whole transformer layer on a subset of rows (dllm_op_layer) against the oracle's
layer, at small sizes spanning several tiles and at the LLaDA-8B width."""
import numpy as np
import pytest
import torch

from oracle.model import OracleModel
from synth import make_weights
from synth.configs import LLADA8B, TINY, DREAM7B, ModelDims, RunConfig

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from token_skip_denoising_b200 import _lib, ops

DEV = "cuda"
TOL_HIDDEN = 2e-2     # max relative error per row, bf16 activations (spec tolerance)


def _rowrel(a, b):
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    return float((np.abs(a - b).max(1) / np.maximum(np.abs(b).max(1), 1e-30)).max())


def _run_layer_case(dims, B, N, rows_per_seq, seed, h_scale=1.0, gain_jitter=0.1, layer_kernel="auto"):
    w = make_weights(dims, seed=seed, device=DEV, gain_jitter=gain_jitter, layers=[0])
    run = RunConfig(name="t", model=dims, batch=B, prompt_len=N - 64 if N > 64 else 0,
                    gen_len=64 if N > 64 else N, block_len=64 if N > 64 else N)
    cfg = _lib.make_config(run, layer_kernel=layer_kernel)
    g = torch.Generator(device=DEV).manual_seed(seed + 1)
    h0 = torch.randn((B * N, dims.d_model), generator=g, device=DEV) * h_scale
    kc0 = torch.randn((B, dims.n_kv_heads, N, dims.head_dim), generator=g, device=DEV).to(torch.bfloat16)
    vc0 = torch.randn(tuple(kc0.shape), generator=g, device=DEV).to(torch.bfloat16)
    rng = np.random.default_rng(seed)
    per = [np.sort(rng.choice(N, rows_per_seq[b], replace=False)) for b in range(B)]
    flat = np.concatenate([b * N + p for b, p in enumerate(per)]).astype(np.int32)
    off = np.concatenate([[0], np.cumsum(rows_per_seq)]).astype(np.int32)
    rows_cap = len(flat)
    cos, sin = ops.rope_table(N, dims.head_dim, dims.rope_theta)
    h = h0.clone()
    kc, vc = kc0.clone(), vc0.clone()
    lw = {k: w[k][0] for k in ("w_qkv", "w_o", "w_gu", "w_down", "g_attn", "g_ffn")}
    ops.layer(cfg, lw, kc, vc, cos, sin, h, torch.tensor(flat, device=DEV),
              torch.tensor([rows_cap], dtype=torch.int32, device=DEV), torch.tensor(off, device=DEV), rows_cap,
              max(rows_per_seq))
    torch.cuda.synchronize()
    # oracle on the same inputs
    wl = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in w.items()}
    om_ = OracleModel(dims, wl)
    K = kc0.cpu().double().numpy()
    V = vc0.cpu().double().numpy()
    b_idx, pos = flat // N, flat % N
    ref = om_.layer(0, h0.cpu().double().numpy()[flat], b_idx, pos, K, V)
    return h, h0, kc, vc, kc0, vc0, flat, ref, K, V


@pytest.mark.parametrize("layer_kernel", ["auto", "split"])   # auto: the fused kernel up to 64 rows
@pytest.mark.parametrize("dims,B,N,rows", [
    (TINY, 1, 64, [8]),
    (TINY, 2, 96, [5, 33]),
    (ModelDims(n_layers=1, d_model=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn_dim=1408, vocab=1024,
               mask_id=1023), 2, 130, [27, 37]),
    (ModelDims(n_layers=1, d_model=512, n_heads=4, n_kv_heads=2, head_dim=128, ffn_dim=1408, vocab=1024,
               mask_id=1023), 3, 130, [1, 70, 130]),
])
def test_layer_matches_oracle(dims, B, N, rows, layer_kernel):
    h, h0, kc, vc, kc0, vc0, flat, ref, K, V = _run_layer_case(dims, B, N, rows, seed=3, layer_kernel=layer_kernel)
    got = h.cpu().double().numpy()
    assert _rowrel(got[flat], ref) < TOL_HIDDEN
    others = np.setdiff1d(np.arange(B * N), flat)
    np.testing.assert_array_equal(got[others], h0.cpu().double().numpy()[others])
    # the recomputed rows' K/V were written; every other cache row is bit-unchanged
    kg, vg = kc.cpu().double().numpy(), vc.cpu().double().numpy()
    for f in others[:50]:
        b, p = divmod(int(f), N)
        assert np.array_equal(kg[b, :, p], kc0[b, :, p].cpu().double().numpy())
    for f in flat:
        b, p = divmod(int(f), N)
        assert _rowrel(kg[b, :, p].reshape(1, -1), K[b, :, p].reshape(1, -1)) < 1e-2
        assert _rowrel(vg[b, :, p].reshape(1, -1), V[b, :, p].reshape(1, -1)) < 1e-2


@pytest.mark.parametrize("dims,N,rows", [(LLADA8B, 768, [7]), (LLADA8B, 768, [32]), (DREAM7B, 1536, [9]),
                                         (LLADA8B, 768, [768]), (DREAM7B, 1536, [1536]), (LLADA8B, 2048, [205])])
def test_layer_full_width(dims, N, rows):
    """LLaDA-8B / Dream-7B layer width with the row counts of the ES skip step, of a refresh
    (every row: 128-wide GEMM tiles and 768 x 768 attention for LLaDA, 256-wide tiles and GQA
    28/4 over 1536 x 1536 for Dream) and of the single-layer microbenchmark at active ratio 0.1."""
    d1 = ModelDims(n_layers=1, d_model=dims.d_model, n_heads=dims.n_heads, n_kv_heads=dims.n_kv_heads,
                   head_dim=dims.head_dim, ffn_dim=dims.ffn_dim, vocab=1024, mask_id=1023,
                   rope_theta=dims.rope_theta)
    h, h0, kc, vc, kc0, vc0, flat, ref, K, V = _run_layer_case(d1, 1, N, rows, seed=5, gain_jitter=0.0)
    got = h.cpu().double().numpy()
    assert _rowrel(got[flat], ref) < TOL_HIDDEN

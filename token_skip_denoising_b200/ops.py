"""Single-kernel entry points (dllm_op_*) on torch CUDA tensors: marshalling only."""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import check, ptr, stream_ptr

EPI_STORE_F32, EPI_STORE_BF16, EPI_RESID_ADD = 0, 1, 3
SEL_TOPK_DESC, SEL_BELOW_CAP_ASC, SEL_FORCED_ASC, SEL_ALL_ELIGIBLE = 0, 1, 2, 3
UNMASK_TOPCONF, UNMASK_CB_DUS = 0, 2

_DEFAULT_WS = 256 << 20


def _ws(nbytes=_DEFAULT_WS):
    """Op workspace: zeroed once (the GEMM tile counters at its start must begin at 0)."""
    return torch.zeros(nbytes, dtype=torch.uint8, device="cuda")


def _L():
    return _lib.load()


def rope_table(N: int, head_dim: int, theta: float):
    c = torch.empty((N, head_dim // 2), dtype=torch.float32, device="cuda")
    s = torch.empty_like(c)
    check(_L().dllm_op_rope_table(ptr(c), ptr(s), N, head_dim, float(theta), stream_ptr()), "rope_table")
    return c, s


def embed_rows(embed, tokens, rows, count, rows_cap, h):
    check(_L().dllm_op_embed_rows(ptr(embed), embed.shape[0], ptr(tokens), ptr(rows), ptr(count), rows_cap,
                                  embed.shape[1], ptr(h), stream_ptr()), "embed_rows")


def rmsnorm_rows(h, g, eps, rows=None, count=None, rows_cap=None, z=None):
    d = h.shape[-1]
    rows_cap = rows_cap if rows_cap is not None else (rows.numel() if rows is not None else h.shape[0])
    if z is None:
        z = torch.empty((rows_cap, d), dtype=torch.bfloat16, device="cuda")
    check(_L().dllm_op_rmsnorm_rows(ptr(h), ptr(rows), ptr(count), rows_cap, d, ptr(g), float(eps), ptr(z),
                                    stream_ptr()), "rmsnorm_rows")
    return z


def gemm(W, X, kind=EPI_STORE_F32, count=None, out=None, rows_map=None, splits=0, bn=0, ws=None):
    """C = X W^T (kind 0 fp32 out, 1 bf16 out, 3 residual add into out[rows_map[j]])."""
    n_out, K = W.shape
    rows_cap = X.shape[0]
    if out is None:
        out = torch.empty((rows_cap, n_out), dtype=torch.float32 if kind == 0 else torch.bfloat16, device="cuda")
    ws = _ws() if ws is None else ws
    check(_L().dllm_op_gemm(kind, ptr(W), n_out, ptr(X), rows_cap, ptr(count), K, ptr(out), ptr(rows_map), splits,
                            bn, ptr(ws), ws.numel(), stream_ptr()), "gemm")
    return out


def qkv_rope(W, X, dims, N, rows_map, rope_cos, rope_sin, kcache, vcache, count=None, splits=0, ws=None):
    rows_cap = X.shape[0]
    q = torch.empty((rows_cap, dims.n_heads * dims.head_dim), dtype=torch.bfloat16, device="cuda")
    ws = _ws() if ws is None else ws
    check(_L().dllm_op_qkv_rope(ptr(W), ptr(X), rows_cap, ptr(count), dims.d_model, dims.n_heads, dims.n_kv_heads,
                                dims.head_dim, N, ptr(rows_map), ptr(rope_cos), ptr(rope_sin), ptr(q), ptr(kcache),
                                ptr(vcache), splits, ptr(ws), ws.numel(), stream_ptr()), "qkv_rope")
    return q


def gate_up(W, X, F, count=None, splits=0, ws=None):
    rows_cap = X.shape[0]
    act = torch.empty((rows_cap, F), dtype=torch.bfloat16, device="cuda")
    ws = _ws() if ws is None else ws
    check(_L().dllm_op_gate_up(ptr(W), F, ptr(X), rows_cap, ptr(count), X.shape[1], ptr(act), splits, ptr(ws),
                               ws.numel(), stream_ptr()), "gate_up")
    return act


def attention(q, kcache, vcache, seq_off, dims, rows_per_seq_cap, splits=0, out=None, ws=None):
    B, Hkv, N, hd = kcache.shape
    rows_cap = q.shape[0]
    out = torch.empty_like(q) if out is None else out
    ws = _ws() if ws is None else ws
    check(_L().dllm_op_attention(ptr(q), ptr(kcache), ptr(vcache), ptr(out), ptr(seq_off), B, rows_cap,
                                 rows_per_seq_cap, N, dims.n_heads, Hkv, hd, splits, ptr(ws), ws.numel(),
                                 stream_ptr()), "attention")
    return out


def lm_head(W, X, mask_id, count=None, out_index=None, n_out=None, ws=None):
    V, d = W.shape
    rows_cap = X.shape[0]
    n = n_out if n_out is not None else rows_cap
    conf = torch.zeros(n, dtype=torch.float32, device="cuda")
    amax = torch.zeros(n, dtype=torch.int32, device="cuda")
    lse = torch.zeros(n, dtype=torch.float32, device="cuda")
    ws = _ws(max(_DEFAULT_WS, rows_cap * (V // 128) * 16 + (64 << 20))) if ws is None else ws
    check(_L().dllm_op_lm_head(ptr(W), V, ptr(X), rows_cap, ptr(count), d, mask_id, ptr(out_index), ptr(conf),
                               ptr(amax), ptr(lse), ptr(ws), ws.numel(), stream_ptr()), "lm_head")
    return conf, amax, lse


def score_es(h, h_prev, conf, alpha, rows=None, n_rows=None, masked_prev=None, tokens=None, mask_id=0, update=0):
    n = n_rows if n_rows is not None else (rows.numel() if rows is not None else h.shape[0])
    score = torch.empty(n, dtype=torch.float32, device="cuda")
    check(_L().dllm_op_score_es(ptr(h), ptr(h_prev), ptr(conf), ptr(masked_prev), ptr(tokens), mask_id, ptr(rows), n,
                                h.shape[-1], float(alpha), update, ptr(score), stream_ptr()), "score_es")
    return score


def score_cos(vnew, vcache, rows, N, n_kv, head_dim, count=None):
    rows_cap = rows.numel()
    sim = torch.empty(rows_cap, dtype=torch.float32, device="cuda")
    check(_L().dllm_op_score_cos(ptr(vnew), ptr(vcache), ptr(rows), ptr(count), rows_cap, N, n_kv, head_dim,
                                 ptr(sim), stream_ptr()), "score_cos")
    return sim


def kl_conf(logits, mask_id, rows=None, zp_store=None, lse_prev=None, has_prev=None, n_pos=None):
    rows_cap, V = logits.shape
    n = n_pos if n_pos is not None else rows_cap
    conf = torch.zeros(n, dtype=torch.float32, device="cuda")
    amax = torch.zeros(n, dtype=torch.int32, device="cuda")
    lse = torch.zeros(n, dtype=torch.float32, device="cuda")
    kl = torch.zeros(rows_cap, dtype=torch.float32, device="cuda")
    check(_L().dllm_op_kl_conf(ptr(logits), ptr(zp_store), ptr(lse_prev), ptr(has_prev), ptr(rows), None, rows_cap,
                               V, mask_id, ptr(conf), ptr(amax), ptr(lse), ptr(kl), stream_ptr()), "kl_conf")
    return conf, amax, lse, kl


def select(scores, B, n, mode, k, tau=0.0, cand_start=0, N=None, lock=None, k_max=None):
    N = N if N is not None else n
    k_max = k_max if k_max is not None else max(1, n if mode == SEL_ALL_ELIGIBLE else min(k, n))
    act = torch.full((B, k_max), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    rows = torch.full((B * n,), -1, dtype=torch.int32, device="cuda")
    off = torch.zeros(B + 1, dtype=torch.int32, device="cuda")
    check(_L().dllm_op_select(ptr(scores), B, n, mode, k, float(tau), cand_start, N, ptr(lock), ptr(act), k_max,
                              ptr(cnt), ptr(rows), ptr(off), stream_ptr()), "select")
    return act, cnt, rows, off


def unmask(tokens, conf, amax, blk_s, blk_len, mask_id, n_commit, round_mask=None, max_out=64,
           mode=UNMASK_TOPCONF, cb_tau=0.0, remain=None):
    B, N = tokens.shape
    pos = torch.full((B, max_out), -1, dtype=torch.int32, device="cuda")
    tok = torch.full((B, max_out), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    check(_L().dllm_op_unmask(ptr(tokens), ptr(conf), ptr(amax), B, N, blk_s, blk_len, mask_id, mode, n_commit,
                              float(cb_tau), ptr(round_mask), ptr(pos), ptr(tok), ptr(cnt), max_out, ptr(remain),
                              stream_ptr()), "unmask")
    return pos, tok, cnt


def layer_workspace_bytes(cfg, rows_cap, rows_per_seq_cap):
    b = ctypes.c_size_t()
    check(_L().dllm_op_layer_workspace(ctypes.byref(cfg), rows_cap, rows_per_seq_cap, ctypes.byref(b)),
          "layer_workspace")
    return b.value


def layer(cfg, lw: dict, kcache, vcache, rope_cos, rope_sin, h, rows, count, seq_off, rows_cap, rows_per_seq_cap,
          ws=None):
    """One transformer layer in place on h[rows[j]] (lw: this layer's weights)."""
    if ws is None:
        ws = torch.zeros(layer_workspace_bytes(cfg, rows_cap, rows_per_seq_cap), dtype=torch.uint8, device="cuda")
    check(_L().dllm_op_layer(ctypes.byref(cfg), ptr(lw["w_qkv"]), ptr(lw["w_o"]), ptr(lw["w_gu"]),
                             ptr(lw["w_down"]), ptr(lw["g_attn"]), ptr(lw["g_ffn"]), ptr(kcache), ptr(vcache),
                             ptr(rope_cos), ptr(rope_sin), ptr(h), ptr(rows), ptr(count), ptr(seq_off), rows_cap,
                             rows_per_seq_cap, ptr(ws), ws.numel(), stream_ptr()), "layer")

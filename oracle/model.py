"""fp64 transformer backbone of the masked diffusion LM (oracle; test infrastructure only).

A pre-norm decoder block without a causal mask:
    h += W_o . Attn(RoPE(W_q z), RoPE(W_k z), W_v z),  z = RMSNorm(h) * g_attn
    h += W_down (silu(W_gate z) * (W_up z)),           z = RMSNorm(h) * g_ffn
and an untied vocabulary projection of RMSNorm(h) * g_final.  The pages use
LLaDA-8B / Dream-7B as-is and describe their denoiser as bidirectional
(ES-dLLM summary sec. 1: full bidirectional attention at every iteration);
the block formulas themselves are the textbook ones and the shapes come from
the workload descriptions.  Only rows that a step recomputes pass through
`layer`; their new K/V rows are written into the cache before attention, and
attention reads all N cached rows of the row's sequence (SureLock summary
sec. 2.1 item 3: locked rows stay visible through their cached K/V).
"""
from __future__ import annotations

import numpy as np
import torch


def to_f64(t) -> np.ndarray:
    """A torch tensor (any dtype, any device) or array as a float64 numpy array."""
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu").double().numpy()


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g, per row."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope_angles(pos: np.ndarray, head_dim: int, theta: float) -> np.ndarray:
    """angle[r, i] = pos[r] * theta^(-2i/hd), i < hd/2."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv = theta ** (-2.0 * i / head_dim)
    return pos.astype(np.float64)[:, None] * inv[None, :]


def apply_rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE on x [m, H, hd]: pairs (i, i + hd/2) rotate by angle[r, i]."""
    hd = x.shape[-1]
    half = hd // 2
    ang = rope_angles(pos, hd, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def softmax_rows(s: np.ndarray) -> np.ndarray:
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Bidirectional attention of m queries over all N keys of one sequence.

    q [m, Hq, hd], K/V [Hkv, N, hd] -> [m, Hq, hd].  Query head j reads KV head
    floor(j * Hkv / Hq); scores are scaled by 1/sqrt(hd); no mask.
    """
    m, hq, hd = q.shape
    hkv = K.shape[0]
    out = np.empty_like(q)
    scale = 1.0 / np.sqrt(hd)
    for j in range(hq):
        kv = (j * hkv) // hq
        s = (q[:, j, :] @ K[kv].T) * scale          # [m, N]
        out[:, j, :] = softmax_rows(s) @ V[kv]
    return out


def lm_confidence(logits: np.ndarray, mask_id: int):
    """Greedy unmasking decision per row.

    tok = argmax over v != mask_id (ties to the lower id); p = softmax over all
    V; conf = p[tok] (the probability of the token the row would commit);
    lse = log-sum-exp of the row.  Returns (conf, tok, lse).
    """
    z = logits
    mx = np.max(z, axis=-1, keepdims=True)
    lse = (mx + np.log(np.sum(np.exp(z - mx), axis=-1, keepdims=True)))[:, 0]
    zm = z.copy()
    zm[:, mask_id] = -np.inf
    tok = np.argmax(zm, axis=-1)
    conf = np.exp(z[np.arange(z.shape[0]), tok] - lse)
    return conf, tok.astype(np.int64), lse


class OracleModel:
    """Weights as fp64 arrays, converted lazily per layer from the synth dict."""

    def __init__(self, dims, weights: dict):
        self.m = dims
        self.w = weights
        self._layer_cache = {}
        self._pos_of = {l: i for i, l in enumerate(weights.get("layers", range(dims.n_layers)))}

    def layer_weights(self, l: int) -> dict:
        if l not in self._layer_cache:
            i = self._pos_of[l]
            w = self.w
            self._layer_cache = {l: {
                "qkv": to_f64(w["w_qkv"][i]), "o": to_f64(w["w_o"][i]),
                "gu": to_f64(w["w_gu"][i]), "down": to_f64(w["w_down"][i]),
                "g_attn": to_f64(w["g_attn"][i]), "g_ffn": to_f64(w["g_ffn"][i]),
            }}
        return self._layer_cache[l]

    def embed(self, tokens: np.ndarray) -> np.ndarray:
        """h0 = E[tok] (no scaling)."""
        e = self.w["embed"]
        idx = torch.as_tensor(np.asarray(tokens, dtype=np.int64), device=e.device)
        return to_f64(e[idx])

    def qkv(self, l: int, h: np.ndarray, pos: np.ndarray):
        """q (after RoPE) [m, Hq, hd], k (after RoPE) and v [m, Hkv, hd]."""
        m = self.m
        lw = self.layer_weights(l)
        z = rmsnorm(h, lw["g_attn"], m.rms_eps)
        y = z @ lw["qkv"].T
        q = y[:, :m.q_dim].reshape(-1, m.n_heads, m.head_dim)
        k = y[:, m.q_dim:m.q_dim + m.kv_dim].reshape(-1, m.n_kv_heads, m.head_dim)
        v = y[:, m.q_dim + m.kv_dim:].reshape(-1, m.n_kv_heads, m.head_dim)
        return apply_rope(q, pos, m.rope_theta), apply_rope(k, pos, m.rope_theta), v

    def value_only(self, l: int, h: np.ndarray) -> np.ndarray:
        """v = W_v RMSNorm(h) [m, Hkv*hd] (the dLLM-Cache similarity probe)."""
        m = self.m
        lw = self.layer_weights(l)
        z = rmsnorm(h, lw["g_attn"], m.rms_eps)
        return z @ lw["qkv"][m.q_dim + m.kv_dim:].T

    def layer(self, l: int, h: np.ndarray, b_idx: np.ndarray, pos: np.ndarray,
              K: np.ndarray, V: np.ndarray) -> np.ndarray:
        """One block for rows (b_idx[r], pos[r]) with hidden h [m, d].

        K, V: this layer's caches [B, Hkv, N, hd], updated in place for the
        given rows before attention.  Returns the block output [m, d].
        """
        m = self.m
        lw = self.layer_weights(l)
        q, k, v = self.qkv(l, h, pos)
        K[b_idx, :, pos, :] = k
        V[b_idx, :, pos, :] = v
        att = np.empty_like(q)
        for b in np.unique(b_idx):
            sel = np.nonzero(b_idx == b)[0]
            att[sel] = attention(q[sel], K[b], V[b])
        h = h + att.reshape(len(pos), m.q_dim) @ lw["o"].T
        z = rmsnorm(h, lw["g_ffn"], m.rms_eps)
        F = m.ffn_dim
        gu = z @ lw["gu"].T
        a = silu(gu[:, :F]) * gu[:, F:]
        return h + a @ lw["down"].T

    def logits(self, h: np.ndarray, chunk: int = 16384) -> np.ndarray:
        """W_lm RMSNorm(h) g_final -> [m, V] (the vocabulary is converted in chunks)."""
        z = rmsnorm(h, to_f64(self.w["g_final"]), self.m.rms_eps)
        W = self.w["lm_head"]
        V = W.shape[0]
        out = np.empty((h.shape[0], V))
        for v0 in range(0, V, chunk):
            out[:, v0:v0 + chunk] = z @ to_f64(W[v0:v0 + chunk]).T
        return out

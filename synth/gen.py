"""Seeded random inputs: weights, prompts and microbenchmark tensors.

Weights are N(0, 0.02) rounded to bf16, norm gains are 1 (optionally jittered
for tests of the gain path), prompt ids are uniform over [0, V-1) so that
the mask id V-1 never appears in a prompt.  Draws use torch generators on the
requested device; the same (seed, device) gives the same values every time.
"""
from __future__ import annotations

import torch

from .configs import ModelDims, RunConfig

WEIGHT_SEED = 0
PROMPT_SEED = 1
MICRO_SEED = 2

_TENSOR_IDS = {"embed": 1, "lm_head": 2, "w_qkv": 3, "w_o": 4, "w_gu": 5, "w_down": 6,
               "g_attn": 7, "g_ffn": 8, "g_final": 9}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, std, seed, device):
    g = _gen(device, seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (x * std).to(torch.bfloat16)


def make_weights(m: ModelDims, seed: int = WEIGHT_SEED, device="cpu", std: float = 0.02,
                 gain_jitter: float = 0.0, layers=None, with_vocab: bool = True) -> dict:
    """All model weights in the library's layout.

    embed, lm_head: [V, d] bf16.  w_qkv: [L, Hq*hd + 2*Hkv*hd, d] (q rows, then k,
    then v).  w_o: [L, d, Hq*hd].  w_gu: [L, 2F, d] (gate rows, then up rows).
    w_down: [L, d, F].  g_attn, g_ffn: [L, d] fp32, g_final: [d] fp32.
    `layers` restricts generation to a subset of layers (others are omitted);
    each layer is drawn from its own seed so a subset equals the full draw.
    with_vocab=False omits the two [V, d] matrices.
    """
    dev = torch.device(device)
    L = m.n_layers
    sel = list(range(L)) if layers is None else list(layers)

    def sd(name, layer=0):
        return seed * 100003 + _TENSOR_IDS[name] * 1009 + layer

    w = {}
    if with_vocab:
        w["embed"] = _normal_bf16((m.vocab, m.d_model), std, sd("embed"), dev)
        w["lm_head"] = _normal_bf16((m.vocab, m.d_model), std, sd("lm_head"), dev)
    shapes = {"w_qkv": (m.qkv_dim, m.d_model), "w_o": (m.d_model, m.q_dim),
              "w_gu": (2 * m.ffn_dim, m.d_model), "w_down": (m.d_model, m.ffn_dim)}
    for name, shp in shapes.items():
        t = torch.empty((len(sel),) + shp, dtype=torch.bfloat16, device=dev)
        for i, l in enumerate(sel):
            t[i] = _normal_bf16(shp, std, sd(name, l), dev)
        w[name] = t
    for name in ("g_attn", "g_ffn"):
        t = torch.ones((len(sel), m.d_model), dtype=torch.float32, device=dev)
        if gain_jitter:
            for i, l in enumerate(sel):
                g = _gen(dev, sd(name, l))
                t[i] += gain_jitter * torch.randn(m.d_model, generator=g, device=dev)
        w[name] = t
    gf = torch.ones(m.d_model, dtype=torch.float32, device=dev)
    if gain_jitter:
        gf += gain_jitter * torch.randn(m.d_model, generator=_gen(dev, sd("g_final")), device=dev)
    w["g_final"] = gf
    w["layers"] = sel
    return w


def make_prompt(cfg: RunConfig, seed: int = PROMPT_SEED) -> torch.Tensor:
    """Prompt ids [B, prompt_len] int32, uniform over [0, V-1) (mask id excluded)."""
    g = _gen("cpu", seed)
    hi = cfg.model.vocab - 1
    return torch.randint(0, hi, (cfg.batch, cfg.prompt_len), generator=g,
                         dtype=torch.int64).to(torch.int32)


def make_tokens(cfg: RunConfig, seed: int = PROMPT_SEED) -> torch.Tensor:
    """Initial sequence [B, N] int32: the prompt followed by gen_len mask ids."""
    p = make_prompt(cfg, seed)
    t = torch.full((cfg.batch, cfg.seq_len), cfg.model.mask_id, dtype=torch.int32)
    t[:, :cfg.prompt_len] = p
    return t


def microbench_hidden(n: int, d: int, seed: int = MICRO_SEED, device="cpu") -> dict:
    """Inputs of the score step at microbenchmark size: two N(0,1) hidden-state
    snapshots [n, d] fp32, previous confidences U(0,1) [n] and a 50% mask flag."""
    g = _gen(device, seed)
    h_cur = torch.randn((n, d), generator=g, device=device)
    h_prev = torch.randn((n, d), generator=g, device=device)
    conf = torch.rand((n,), generator=g, device=device)
    masked_prev = (torch.rand((n,), generator=g, device=device) < 0.5).to(torch.uint8)
    return {"h_cur": h_cur, "h_prev": h_prev, "conf": conf, "masked_prev": masked_prev}


def microbench_active(n: int, k: int, pattern: str, seed: int = MICRO_SEED) -> torch.Tensor:
    """Ascending active indices [k] int32: 'random' (uniform without replacement)
    or 'contiguous' (one span of k rows at a seeded 32-aligned offset)."""
    g = _gen("cpu", seed + 17)
    if pattern == "random":
        idx = torch.randperm(n, generator=g)[:k]
        return torch.sort(idx).values.to(torch.int32)
    if pattern == "contiguous":
        slots = max(1, (n - k) // 32 + 1)
        off = int(torch.randint(0, slots, (1,), generator=g)) * 32
        off = min(off, n - k)
        return torch.arange(off, off + k, dtype=torch.int32)
    raise ValueError(pattern)


def kv_cache_fill(n_layers: int, batch: int, n_kv: int, n: int, hd: int,
                  seed: int = MICRO_SEED, device="cpu") -> torch.Tensor:
    """A pre-filled K/V cache [L, 2, B, Hkv, N, hd] bf16, N(0,1)."""
    g = _gen(device, seed + 31)
    x = torch.randn((n_layers, 2, batch, n_kv, n, hd), generator=g, device=device)
    return x.to(torch.bfloat16)


def lock_pattern(batch: int, n: int, frac: float, seed: int = MICRO_SEED) -> torch.Tensor:
    """A seeded lock pattern [B, N] uint8: exactly round(frac * N) positions of each
    sequence marked, drawn uniformly without replacement (the forced lock fraction of
    the SureLock measurement mode)."""
    g = _gen("cpu", seed + 53)
    out = torch.zeros((batch, n), dtype=torch.uint8)
    m = int(round(frac * n))
    for b in range(batch):
        out[b, torch.randperm(n, generator=g)[:m]] = 1
    return out

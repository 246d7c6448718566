"""The seeded input recipe both sides draw from (no GPU): shapes and layout of the weights,
their distribution, the prompt / mask layout of the initial sequence, the microbenchmark
tensors, and that a seed always gives the same values."""
import math

import numpy as np
import torch

from synth import get_config, lock_pattern, make_tokens, make_weights
from synth.configs import ModelDims
from synth.gen import kv_cache_fill, microbench_active, microbench_hidden

DIMS = ModelDims(n_layers=3, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn_dim=512, vocab=1024,
                 mask_id=1023)


def test_weight_layout_and_distribution():
    w = make_weights(DIMS)
    L, d, F, V = DIMS.n_layers, DIMS.d_model, DIMS.ffn_dim, DIMS.vocab
    qkv = (DIMS.n_heads + 2 * DIMS.n_kv_heads) * DIMS.head_dim
    shapes = {"embed": (V, d), "lm_head": (V, d), "w_qkv": (L, qkv, d), "w_o": (L, d, DIMS.n_heads * DIMS.head_dim),
              "w_gu": (L, 2 * F, d), "w_down": (L, d, F), "g_attn": (L, d), "g_ffn": (L, d), "g_final": (d,)}
    for k, shp in shapes.items():
        assert tuple(w[k].shape) == shp, k
        assert w[k].dtype == (torch.float32 if k.startswith("g_") else torch.bfloat16), k
    for k in ("embed", "lm_head", "w_qkv", "w_o", "w_gu", "w_down"):
        x = w[k].float()
        n = x.numel()
        assert abs(float(x.mean())) < 5 * 0.02 / math.sqrt(n)         # zero mean
        assert abs(float(x.std()) - 0.02) < 0.02 * 0.05                # std 0.02 (bf16-rounded)
    for k in ("g_attn", "g_ffn", "g_final"):
        assert torch.all(w[k] == 1)                                    # gains 1 unless jittered
    assert not torch.equal(w["w_qkv"][0], w["w_qkv"][1])               # every layer its own draw
    assert not torch.equal(w["embed"], w["lm_head"])                   # untied


def test_a_layer_subset_equals_the_full_draw():
    full, sub = make_weights(DIMS), make_weights(DIMS, layers=[2])
    for k in ("w_qkv", "w_o", "w_gu", "w_down"):
        assert torch.equal(sub[k][0], full[k][2]), k
    assert torch.equal(make_weights(DIMS)["w_o"], full["w_o"])          # same seed, same values
    assert not torch.equal(make_weights(DIMS, seed=5)["w_o"], full["w_o"])


def test_initial_sequence_is_prompt_then_mask_ids():
    for name in ("tiny", "llada_es", "dream_surelock", "llada_cache_dus"):
        cfg = get_config(name)
        t = make_tokens(cfg)
        assert t.dtype == torch.int32 and tuple(t.shape) == (cfg.batch, cfg.prompt_len + cfg.gen_len)
        prompt, gen = t[:, :cfg.prompt_len], t[:, cfg.prompt_len:]
        assert torch.all(gen == cfg.model.mask_id)
        if cfg.prompt_len:
            assert int(prompt.min()) >= 0 and int(prompt.max()) < cfg.model.vocab - 1   # mask id never in a prompt
        assert torch.equal(make_tokens(cfg), t)
    cfg = get_config("llada_es")
    p = make_tokens(cfg)[:, :cfg.prompt_len].numpy().ravel()
    # uniform over [0, V-1): the mean of 512 draws sits near (V-2)/2
    assert abs(p.mean() - (cfg.model.vocab - 2) / 2) < 4 * cfg.model.vocab / math.sqrt(12 * p.size)


def test_microbenchmark_tensors():
    hin = microbench_hidden(4096, 64)
    assert abs(float(hin["h_cur"].std()) - 1) < 0.02 and abs(float(hin["conf"].mean()) - 0.5) < 0.02
    assert abs(float(hin["masked_prev"].float().mean()) - 0.5) < 0.03
    for pattern in ("random", "contiguous"):
        a = microbench_active(2048, 205, pattern).numpy()
        assert a.dtype == np.int32 and len(a) == 205 and np.all(np.diff(a) > 0) and a[-1] < 2048
    c = microbench_active(2048, 205, "contiguous").numpy()
    assert c[0] % 32 == 0 and np.all(np.diff(c) == 1)
    kv = kv_cache_fill(2, 1, 2, 64, 32)
    assert tuple(kv.shape) == (2, 2, 1, 2, 64, 32) and kv.dtype == torch.bfloat16
    lp = lock_pattern(3, 100, 0.25)
    assert lp.dtype == torch.uint8 and torch.all(lp.sum(dim=1) == 25)

"""Pins of the oracle's transformer backbone against closed forms, brute force and
invariants that do not reuse the oracle's own formulas."""
import math

import numpy as np
import pytest
import torch

from oracle.model import (OracleModel, apply_rope, attention, lm_confidence, rmsnorm,
                          silu)
from synth.configs import ModelDims

RNG = np.random.default_rng(1234)


def test_rmsnorm_closed_form():
    # x = (3, 4): mean square = 12.5; with eps = 0.5 the divisor is sqrt(13)
    out = rmsnorm(np.array([[3.0, 4.0]]), np.array([1.0, 2.0]), 0.5)
    np.testing.assert_allclose(out, [[3 / math.sqrt(13), 8 / math.sqrt(13)]], rtol=1e-15)
    # a constant row c maps to c / sqrt(c^2 + eps)
    c = 0.25
    out = rmsnorm(np.full((1, 8), c), np.ones(8), 1e-5)
    np.testing.assert_allclose(out, c / math.sqrt(c * c + 1e-5), rtol=1e-15)


def test_rope_hand_rotation():
    # hd = 4, theta = 100: frequencies 1 and 100^(-1/2) = 0.1; position 2 -> angles 2 and 0.2
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    out = apply_rope(x, np.array([2]), 100.0)[0, 0]
    a0, a1 = 2.0, 0.2
    exp = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
           3 * math.cos(a0) + 1 * math.sin(a0), 4 * math.cos(a1) + 2 * math.sin(a1)]
    np.testing.assert_allclose(out, exp, rtol=1e-14)
    # position 0 is the identity
    np.testing.assert_array_equal(apply_rope(x, np.array([0]), 100.0), x)


def test_rope_norm_and_relative_position():
    hd = 64
    q = RNG.standard_normal((1, 1, hd))
    k = RNG.standard_normal((1, 1, hd))
    for p in (0, 7, 300):
        r = apply_rope(q, np.array([p]), 10000.0)
        assert np.linalg.norm(r) == pytest.approx(np.linalg.norm(q), rel=1e-13)
    dots = []
    for shift in (0, 5, 1000):
        rq = apply_rope(q, np.array([11 + shift]), 10000.0)
        rk = apply_rope(k, np.array([4 + shift]), 10000.0)
        dots.append(float(np.sum(rq * rk)))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)


def _brute_attention(q, K, V):
    """Explicit loops with math.exp; query head j reads kv head j // (Hq / Hkv)."""
    m, hq, hd = q.shape
    hkv, n, _ = K.shape
    grp = hq // hkv
    out = np.zeros_like(q)
    for r in range(m):
        for j in range(hq):
            kv = j // grp
            s = [sum(q[r, j, t] * K[kv, i, t] for t in range(hd)) / math.sqrt(hd) for i in range(n)]
            mx = max(s)
            e = [math.exp(v - mx) for v in s]
            z = sum(e)
            for t in range(hd):
                out[r, j, t] = sum(e[i] * V[kv, i, t] for i in range(n)) / z
    return out


@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (6, 3)])
def test_attention_brute_force(hq, hkv):
    q = RNG.standard_normal((3, hq, 4))
    K = RNG.standard_normal((hkv, 5, 4))
    V = RNG.standard_normal((hkv, 5, 4))
    np.testing.assert_allclose(attention(q, K, V), _brute_attention(q, K, V), rtol=1e-12, atol=1e-14)


def test_attention_special_cases():
    q = RNG.standard_normal((2, 2, 8))
    V = RNG.standard_normal((2, 6, 8))
    # identical keys -> uniform weights -> mean of the values
    K = np.repeat(RNG.standard_normal((2, 1, 8)), 6, axis=1)
    np.testing.assert_allclose(attention(q, K, V), np.broadcast_to(V.mean(axis=1)[None], (2, 2, 8)),
                               rtol=1e-12)
    # a single key returns its value exactly
    out = attention(q, K[:, :1], V[:, :1])
    np.testing.assert_allclose(out, np.broadcast_to(V[:, 0][None], (2, 2, 8)), rtol=1e-15)


def test_silu_values():
    assert silu(np.array(0.0)) == 0.0
    np.testing.assert_allclose(silu(np.array([1.0, -2.0])),
                               [1 / (1 + math.exp(-1)), -2 / (1 + math.exp(2))], rtol=1e-15)


def test_lm_confidence_closed_form():
    # logits ln(1), ln(2), ln(5) over V = 3 -> p = (1/8, 2/8, 5/8); mask id 2 excluded from argmax
    z = np.log(np.array([[1.0, 2.0, 5.0]]))
    conf, tok, lse = lm_confidence(z, mask_id=2)
    assert tok[0] == 1
    assert conf[0] == pytest.approx(2 / 8, rel=1e-14)
    assert lse[0] == pytest.approx(math.log(8), rel=1e-14)
    # ties go to the lower id
    conf, tok, _ = lm_confidence(np.array([[0.5, 2.0, 2.0, 1.0]]), mask_id=0)
    assert tok[0] == 1
    # the mask id never wins even when largest
    conf, tok, _ = lm_confidence(np.array([[9.0, 1.0, 0.0]]), mask_id=0)
    assert tok[0] == 1


def _tiny_dims(hq=2, hkv=2, d=8, hd=4, F=6):
    return ModelDims(n_layers=1, d_model=d, n_heads=hq, n_kv_heads=hkv, head_dim=hd,
                     ffn_dim=F, vocab=16, mask_id=15, rope_theta=10000.0, rms_eps=1e-6)


def _rand_weights(m, seed=0):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: (torch.randn(*s, generator=g) * 0.3).to(torch.bfloat16)
    return {"embed": r(m.vocab, m.d_model), "lm_head": r(m.vocab, m.d_model),
            "w_qkv": r(1, m.qkv_dim, m.d_model), "w_o": r(1, m.d_model, m.q_dim),
            "w_gu": r(1, 2 * m.ffn_dim, m.d_model), "w_down": r(1, m.d_model, m.ffn_dim),
            "g_attn": torch.ones(1, m.d_model), "g_ffn": torch.ones(1, m.d_model),
            "g_final": torch.ones(m.d_model), "layers": [0]}


def _run_layer(m, w, h, pos, n):
    om = OracleModel(m, w)
    K = np.zeros((1, 1, m.n_kv_heads, n, m.head_dim))
    V = np.zeros_like(K)
    b = np.zeros(len(pos), dtype=np.int64)
    return om.layer(0, h, b, np.asarray(pos), K[0], V[0]), K, V


def test_layer_is_identity_without_output_projections():
    m = _tiny_dims()
    w = _rand_weights(m)
    w["w_o"].zero_()
    w["w_down"].zero_()
    h = RNG.standard_normal((3, m.d_model))
    out, _, _ = _run_layer(m, w, h, [0, 1, 2], 3)
    np.testing.assert_array_equal(out, h)


def test_qkv_scores_depend_on_relative_position_only():
    # RoPE must rotate both q and k with the row's position: shifting every position by
    # a constant leaves all attention scores q_i . k_j unchanged
    m = _tiny_dims()
    om = OracleModel(m, _rand_weights(m, 1))
    h = RNG.standard_normal((4, m.d_model))
    q0, k0, _ = om.qkv(0, h, np.array([0, 1, 2, 3]))
    q1, k1, _ = om.qkv(0, h, np.array([30, 31, 32, 33]))
    s0 = np.einsum("ihd,jhd->hij", q0, k0)
    s1 = np.einsum("ihd,jhd->hij", q1, k1)
    np.testing.assert_allclose(s0, s1, rtol=1e-10, atol=1e-12)
    assert not np.allclose(q0, q1)


def test_gqa_equals_mha_with_duplicated_kv_heads():
    mg = _tiny_dims(hq=4, hkv=2, d=16)
    mm = _tiny_dims(hq=4, hkv=4, d=16)
    wg = _rand_weights(mg, 2)
    wm = dict(wg)
    qd, hd = mg.q_dim, mg.head_dim
    kv = wg["w_qkv"][0]
    k_rows = kv[qd:qd + 2 * hd].reshape(2, hd, -1)
    v_rows = kv[qd + 2 * hd:].reshape(2, hd, -1)
    dup = lambda t: t.repeat_interleave(2, dim=0).reshape(4 * hd, -1)
    wm["w_qkv"] = torch.cat([kv[:qd], dup(k_rows), dup(v_rows)], 0)[None]
    h = RNG.standard_normal((3, mg.d_model))
    a, _, _ = _run_layer(mg, wg, h, [0, 1, 2], 3)
    b, _, _ = _run_layer(mm, wm, h, [0, 1, 2], 3)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def test_ffn_scalar_closed_form():
    # d = 1, F = 1, attention removed: out = h + wd * silu(wg z) * (wu z), z = h / sqrt(h^2 + eps)
    m = ModelDims(n_layers=1, d_model=1, n_heads=1, n_kv_heads=1, head_dim=2, ffn_dim=1,
                  vocab=4, mask_id=3, rms_eps=1e-6)
    w = {"w_qkv": torch.zeros(1, 6, 1), "w_o": torch.zeros(1, 1, 2),
         "w_gu": torch.tensor([[[0.5], [-1.5]]]), "w_down": torch.tensor([[[2.0]]]),
         "g_attn": torch.ones(1, 1), "g_ffn": torch.ones(1, 1), "g_final": torch.ones(1),
         "embed": torch.zeros(4, 1), "lm_head": torch.zeros(4, 1), "layers": [0]}
    h = np.array([[0.7]])
    out, _, _ = _run_layer(m, w, h, [0], 1)
    z = 0.7 / math.sqrt(0.49 + 1e-6)
    g = 0.5 * z
    exp = 0.7 + 2.0 * (g / (1 + math.exp(-g))) * (-1.5 * z)
    assert out[0, 0] == pytest.approx(exp, rel=1e-14)


def test_layer_writes_kv_before_attention():
    # one row over a one-slot cache attends only to itself, so with the FFN output
    # projection removed the block adds exactly W_o v (softmax over a single key is 1)
    m = _tiny_dims()
    w = _rand_weights(m, 3)
    w["w_down"].zero_()
    h = RNG.standard_normal((1, m.d_model))
    out, K, V = _run_layer(m, w, h, [0], 1)
    om = OracleModel(m, w)
    _, k, v = om.qkv(0, h, np.array([0]))
    np.testing.assert_array_equal(K[0, 0, :, 0, :], k[0])
    np.testing.assert_array_equal(V[0, 0, :, 0, :], v[0])
    wo = w["w_o"][0].double().numpy()
    np.testing.assert_allclose(out - h, v.reshape(1, -1) @ wo.T, rtol=1e-12, atol=1e-14)

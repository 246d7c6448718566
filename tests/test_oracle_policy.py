"""Pins of the oracle's scores, selection rules and the DUS schedule."""
import json
import math
import os

import numpy as np
import pytest
import scipy.spatial.distance
import scipy.stats

from oracle.policy import (cosine_rows, dus_num_rounds, dus_rounds, dus_schedule,
                           es_importance, kl_from_logits, threshold_cap_select, topk_select,
                           unmask_cb_dus, unmask_topconf)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(99)


# ---------------------------------------------------------------- Eq. 1

def test_es_importance_hand_computed():
    # d = 4 so sqrt(d) = 2.
    # row 0: H_prev = (1,0,0,0) (norm 1), H_cur = (1,1,0,0): L1 diff 1 -> var 1/2
    # row 1: H_prev = (0,3,4,0) (norm 5), H_cur = (0,3,4,0): var 0
    # row 2: H_prev = (2,2,2,2) (norm 4), H_cur = (0,0,0,0): L1 diff 8 -> var 8/(2*4) = 1
    h_prev = np.array([[1, 0, 0, 0], [0, 3, 4, 0], [2, 2, 2, 2]], dtype=float)
    h_cur = np.array([[1, 1, 0, 0], [0, 3, 4, 0], [0, 0, 0, 0]], dtype=float)
    c = np.array([0.2, 0.9, 0.0])
    out = es_importance(0.5, c, h_cur, h_prev)
    np.testing.assert_allclose(out, [0.5 * 0.2 + 0.5 * 0.5, 0.5 * 0.9, 0.5 * 1.0], rtol=1e-15)
    out = es_importance(0.25, c, h_cur, h_prev)
    np.testing.assert_allclose(out, [0.05 + 0.375, 0.225, 0.75], rtol=1e-15)


def test_es_importance_limits_and_invariances():
    h_prev = RNG.standard_normal((5, 16))
    h_cur = RNG.standard_normal((5, 16))
    c = RNG.random(5)
    np.testing.assert_array_equal(es_importance(1.0, c, h_cur, h_prev), c)        # alpha = 1 -> I = c
    np.testing.assert_array_equal(es_importance(0.3, c, h_prev, h_prev), 0.3 * c)  # no change -> var 0
    a = es_importance(0.0, c, h_cur, h_prev)
    b = es_importance(0.0, c, 7.5 * h_cur, 7.5 * h_prev)                          # scale-free variation
    np.testing.assert_allclose(a, b, rtol=1e-13)
    z = es_importance(0.5, c, h_cur, np.zeros_like(h_prev))                      # zero previous state
    np.testing.assert_array_equal(z, 0.5 * c)


# ---------------------------------------------------------------- KL

def _lse(z):
    m = z.max(axis=-1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=-1))


def test_kl_against_scipy_entropy():
    z_t = RNG.standard_normal((6, 50)) * 2
    z_p = RNG.standard_normal((6, 50)) * 2
    d = kl_from_logits(z_t, _lse(z_t), z_p, _lse(z_p))
    for i in range(6):
        p = np.exp(z_t[i] - _lse(z_t[i:i + 1])[0])
        q = np.exp(z_p[i] - _lse(z_p[i:i + 1])[0])
        assert d[i] == pytest.approx(scipy.stats.entropy(p, q), rel=1e-10)
    assert np.all(d >= 0)


def test_kl_two_point_closed_form_and_identity():
    a, b = 0.8, 0.3
    z_t = np.log(np.array([[a, 1 - a]]))
    z_p = np.log(np.array([[b, 1 - b]]))
    d = kl_from_logits(z_t, _lse(z_t), z_p, _lse(z_p))[0]
    assert d == pytest.approx(a * math.log(a / b) + (1 - a) * math.log((1 - a) / (1 - b)), rel=1e-13)
    z = RNG.standard_normal((4, 100))
    assert np.all(kl_from_logits(z, _lse(z), z, _lse(z)) == 0.0)   # identical distributions: exactly 0


# ---------------------------------------------------------------- cosine

def test_cosine_against_scipy_and_zero_cases():
    a = RNG.standard_normal((5, 12))
    b = RNG.standard_normal((5, 12))
    s = cosine_rows(a, b)
    for i in range(5):
        assert s[i] == pytest.approx(1 - scipy.spatial.distance.cosine(a[i], b[i]), rel=1e-12)
    z = np.zeros((1, 12))
    assert cosine_rows(z, z)[0] == 1.0
    assert cosine_rows(a[:1], z)[0] == 0.0
    assert cosine_rows(a[:1], 3 * a[:1])[0] == pytest.approx(1.0, rel=1e-15)


# ---------------------------------------------------------------- selection

def _check_topk(scores, k, sel):
    n = len(scores)
    assert len(sel) == min(k, n)
    assert list(sel) == sorted(set(sel))
    chosen = np.zeros(n, bool)
    chosen[sel] = True
    s32 = scores.astype(np.float32)
    for i in range(n):
        for j in range(n):
            if chosen[i] and not chosen[j]:
                # every chosen row ranks above every dropped row under (score desc, index asc)
                assert s32[i] > s32[j] or (s32[i] == s32[j] and i < j)


@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (32, 7), (33, 33), (100, 25), (64, 0)])
def test_topk_select_properties(n, k):
    for trial in range(5):
        scores = RNG.integers(0, 4, n).astype(float) / 4.0 if trial % 2 else RNG.random(n)
        _check_topk(scores, k, topk_select(scores, k))


def test_topk_select_brute_force_small():
    # exhaustive over all 3^5 score vectors with ties
    import itertools
    for vals in itertools.product([0.0, 0.5, 1.0], repeat=5):
        s = np.array(vals)
        for k in range(6):
            _check_topk(s, k, topk_select(s, k))


def test_topk_select_nan_and_signed_zero():
    s = np.array([np.nan, -0.0, 0.0, -1.0])
    assert list(topk_select(s, 2)) == [1, 2]     # -0 ranks as +0, lower index first
    assert list(topk_select(s, 4)) == [0, 1, 2, 3]
    assert list(topk_select(s, 3)) == [1, 2, 3]  # NaN last


def test_threshold_cap_select_properties():
    for trial in range(20):
        n = int(RNG.integers(1, 60))
        sims = np.round(RNG.random(n) * 4) / 4
        tau, cap = 0.6, int(RNG.integers(0, n + 1))
        sel = threshold_cap_select(sims, tau, cap)
        below = np.nonzero(sims < tau)[0]
        assert len(sel) == min(cap, len(below))
        assert set(sel) <= set(below)
        assert list(sel) == sorted(sel)
        dropped = sorted(set(below) - set(sel))
        for i in sel:
            for j in dropped:
                assert sims[i] < sims[j] or (sims[i] == sims[j] and i < j)
        forced = threshold_cap_select(sims, -1.0, cap, forced=True)
        assert len(forced) == min(cap, n)


def test_unmask_topconf_properties():
    conf = np.array([0.1, 0.9, 0.9, 0.3, 0.95, 0.2])
    masked = np.array([True, True, True, True, False, True])
    assert list(unmask_topconf(conf, masked, 2)) == [1, 2]     # 0.95 is not masked; tie -> lower pos
    assert list(unmask_topconf(conf, masked, 1)) == [1]
    assert list(unmask_topconf(conf, masked, 10)) == [0, 1, 2, 3, 5]


def test_unmask_cb_dus_hand_example():
    # confidences by position:       0     1     2     3     4     5
    conf = np.array([0.90, 0.95, 0.20, 0.85, 0.99, 0.50])
    masked = np.ones(6, bool)
    # 4 (0.99) taken, 3 and 5 blocked; 1 (0.95) taken, 0 and 2 blocked; 0 and 3 skipped; 5 < tau: stop
    assert list(unmask_cb_dus(conf, masked, 0.8, 4)) == [1, 4]
    assert list(unmask_cb_dus(conf, masked, 0.8, 1)) == [4]                   # cap
    assert list(unmask_cb_dus(conf, masked, 0.999, 4)) == [4]                 # the first is always taken
    assert list(unmask_cb_dus(conf, masked, -1.0, 6)) == [1, 4]               # 0, 2, 3, 5 all blocked
    m2 = masked.copy()
    m2[4] = False                                                              # 4 already unmasked
    assert list(unmask_cb_dus(conf, m2, 0.8, 4)) == [1, 3]                    # 1; 0 blocked; 3
    assert list(unmask_cb_dus(np.array([0.5, 0.5, 0.5]), np.ones(3, bool), 0.0, 3)) == [0, 2]   # ties: lower first


def test_unmask_cb_dus_properties():
    rng = np.random.default_rng(7)
    for trial in range(300):
        n = int(rng.integers(1, 40))
        conf = rng.random(n).astype(np.float32)
        conf[rng.random(n) < 0.1] = rng.choice(conf)                           # ties
        masked = rng.random(n) < 0.7
        if not masked.any():
            masked[int(rng.integers(n))] = True
        tau = float(rng.choice([0.0, 0.3, 0.7, 0.95, 2.0]))
        cap = int(rng.integers(1, 8))
        got = list(unmask_cb_dus(conf, masked, tau, cap))
        assert 1 <= len(got) <= cap and all(masked[i] for i in got)
        assert all(b - a >= 2 for a, b in zip(got, got[1:]))                   # mutually non-adjacent
        order = sorted(np.nonzero(masked)[0], key=lambda i: (-conf[i], i))
        assert got[0] == order[0] or order[0] in got                           # the best is always taken
        assert sum(conf[i] < np.float32(tau) for i in got) <= 1                # only the forced first may be below
        if len(got) < cap:
            # maximal: a qualifying position left out is next to a taken one of higher priority
            rank = {i: r for r, i in enumerate(order)}
            for i in order:
                if i in got or conf[i] < np.float32(tau):
                    continue
                assert any(abs(i - j) == 1 and rank[j] < rank[i] for j in got), (conf, masked, tau, cap, got)


# ---------------------------------------------------------------- DUS

def test_dus_matches_hallway_example():
    g = json.load(open(os.path.join(GOLDEN, "dus_hallway.json")))
    rounds = dus_rounds(g["length"], g["rounds"])
    assert [list(r + 1) for r in rounds] == g["expected_1_indexed"]


def test_dus_round_count():
    g = json.load(open(os.path.join(GOLDEN, "dus_rounds.json")))
    for b, r in g["cases"].items():
        assert dus_num_rounds(int(b)) == r
        assert len(dus_schedule(int(b))) == r


@pytest.mark.parametrize("block", [1, 3, 4, 5, 8, 16, 31, 32, 64, 100, 128])
def test_dus_partition_and_non_adjacency(block):
    rounds = dus_schedule(block)
    assert len(rounds) == max(1, math.ceil(math.log2(block))) if block > 1 else len(rounds) == 1
    allp = np.concatenate(rounds)
    assert sorted(allp.tolist()) == list(range(block))           # a partition of the block
    for r in rounds:
        assert len(r) > 0
        assert np.all(np.diff(np.sort(r)) >= 2)                   # mutually non-adjacent
    if block >= 4 and block & (block - 1) == 0:
        # power-of-two block, coarse to fine: 2, 2, 4, 8, ..., B/2 positions per round
        sizes = [len(r) for r in rounds]
        assert sizes == [2] + [2 ** i for i in range(1, len(rounds))]


def test_dus_rejects_block_of_two():
    with pytest.raises(ValueError):
        dus_schedule(2)

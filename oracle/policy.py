"""Row scores, row selection and unmasking rules (oracle; test infrastructure only).

Each function follows one passage of the pages; where they leave a detail
open, the docstring states the reading taken.
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------- scores

def es_importance(alpha: float, c_prev: np.ndarray, h_cur: np.ndarray,
                  h_prev: np.ndarray) -> np.ndarray:
    """ES-dLLM importance, Eq. 1 (ES-dLLM summary, sec. 2.1):

        I_i = alpha * c_i + (1 - alpha) * ||H_t,i - H_t-1,i||_1 / (sqrt(d) * ||H_t-1,i||_2)

    c_prev [n], h_cur / h_prev [n, d].  A row whose previous hidden state has
    zero norm gets variation 0 (the pages are silent on that case).
    """
    d = h_cur.shape[-1]
    l1 = np.sum(np.abs(h_cur - h_prev), axis=-1)
    l2 = np.sqrt(np.sum(h_prev * h_prev, axis=-1))
    var = np.zeros_like(l1)
    nz = l2 > 0
    var[nz] = l1[nz] / (math.sqrt(d) * l2[nz])
    return alpha * c_prev + (1.0 - alpha) * var


def kl_from_logits(z_t: np.ndarray, lse_t: np.ndarray, z_p: np.ndarray,
                   lse_p: np.ndarray) -> np.ndarray:
    """SureLock local divergence D = KL(p_t || p_t-1) per row (SureLock summary,
    sec. 2.1 item 1), from logits and their log-sum-exp:

        D = sum_v p_t(v) * [(z_t(v) - lse_t) - (z_t-1(v) - lse_t-1)],  clamped at 0.
    """
    p = np.exp(z_t - lse_t[:, None])
    d = np.sum(p * ((z_t - lse_t[:, None]) - (z_p - lse_p[:, None])), axis=-1)
    return np.maximum(d, 0.0)


def cosine_rows(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Per-row cosine similarity; 1 when both rows are zero, 0 when one is."""
    dot = np.sum(a * b, axis=-1)
    na = np.sqrt(np.sum(a * a, axis=-1))
    nb = np.sqrt(np.sum(b * b, axis=-1))
    out = np.zeros_like(dot)
    both = (na > 0) & (nb > 0)
    out[both] = dot[both] / (na[both] * nb[both])
    out[(na == 0) & (nb == 0)] = 1.0
    return out


# ---------------------------------------------------------------- selection

def canonical_score(x) -> float:
    """Scores are ranked as float32 values; -0 ranks as +0 and NaN below -inf."""
    v = float(np.float32(x))
    if math.isnan(v):
        return -math.inf, 1
    return (v + 0.0), 0


def _key_desc(score, i):
    v, nan = canonical_score(score)
    return (nan, -v, i)


def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """ES-dLLM early skip (ES-dLLM summary, sec. 2.1 item 2): keep the k rows with
    the highest score.  Ties go to the lower index; NaN ranks last.  The result
    is in ascending index order."""
    n = len(scores)
    k = max(0, min(k, n))
    order = sorted(range(n), key=lambda i: _key_desc(scores[i], i))
    return np.array(sorted(order[:k]), dtype=np.int64)


def threshold_cap_select(sims: np.ndarray, tau: float, cap: int,
                         forced: bool = False) -> np.ndarray:
    """dLLM-Cache partial update (dLLM-Cache explainer, sec. 3): rows whose
    similarity to their cached features is below tau are recomputed, at most
    `cap` of them (the lowest similarities; ties to the lower index).  With
    forced=True exactly min(cap, n) lowest rows are taken regardless of tau.
    Ascending index order."""
    n = len(sims)

    def key(i):
        v, nan = canonical_score(sims[i])
        return (1 - nan, v, i)   # NaN counts as most dissimilar

    if forced:
        cand = list(range(n))
    else:
        cand = [i for i in range(n) if math.isnan(float(sims[i])) or float(np.float32(sims[i])) < tau]
    cand.sort(key=key)
    return np.array(sorted(cand[:max(0, min(cap, n))]), dtype=np.int64)


def unmask_topconf(conf: np.ndarray, masked: np.ndarray, n: int) -> np.ndarray:
    """Commit the n masked positions with the highest confidence (ES-dLLM summary,
    sec. 1: a few high-confidence tokens are unmasked per step).  conf and
    masked are over the candidate positions; ties go to the lower position.
    Returns ascending positions (fewer than n when fewer are masked)."""
    cand = [i for i in range(len(conf)) if masked[i]]
    cand.sort(key=lambda i: _key_desc(conf[i], i))
    return np.array(sorted(cand[:n]), dtype=np.int64)


def unmask_cb_dus(conf: np.ndarray, masked: np.ndarray, tau: float, cap: int) -> np.ndarray:
    """Confidence-bounded unmasking with the dilation principle of DUS as a post-filter
    (Plan for Speed summary, sec. 3 'complementary hybrid extension': spacing applied to an
    adaptive, confidence-bounded sampler keeps it from picking densely clustered tokens).
    Masked positions are taken in order of confidence (descending, ties to the lower
    position) while their confidence is at least tau -- the first one always, so every step
    unmasks something -- skipping any position next to one already taken in this step, at
    most `cap` in all.  Confidences and tau compare as float32.  Ascending positions."""
    tau32 = float(np.float32(tau))
    order = sorted((i for i in range(len(conf)) if masked[i]), key=lambda i: _key_desc(conf[i], i))
    taken, blocked = [], set()
    for i in order:
        if len(taken) >= cap:
            break
        v, nan = canonical_score(conf[i])
        if taken and (nan or not v >= tau32):
            break                      # confidences only fall from here on
        if i in blocked:
            continue
        taken.append(i)
        blocked.update((i - 1, i + 1))
    return np.array(sorted(taken), dtype=np.int64)


# ---------------------------------------------------------------- DUS

def dus_rounds(length: int, n_rounds: int, base: int = 2):
    """Dilated groups over positions 0..length-1 (Plan for Speed summary, sec. 2):
    round r takes the positions divisible by base^(R-1-r) that no earlier
    round took, so the first rounds are sparse and the last fills the gaps.
    With base 2 every round is mutually non-adjacent."""
    taken = np.zeros(length, dtype=bool)
    rounds = []
    for r in range(n_rounds):
        stride = base ** (n_rounds - 1 - r)
        sel = [p for p in range(length) if p % stride == 0 and not taken[p]]
        taken[sel] = True
        rounds.append(np.array(sel, dtype=np.int64))
    return rounds


def dus_num_rounds(block: int, base: int = 2) -> int:
    """R = ceil(log_a B) (Plan for Speed summary, sec. 2); one round for B = 1."""
    if block <= 1:
        return 1
    r = 0
    while base ** r < block:
        r += 1
    return r


def dus_schedule(block: int, base: int = 2):
    """The rounds of one block of size B.  B = 2 cannot be split into
    non-adjacent groups in ceil(log2 2) = 1 round and is rejected."""
    if block == 2:
        raise ValueError("DUS: a block of 2 has no non-adjacent single-round schedule")
    return dus_rounds(block, dus_num_rounds(block, base), base)

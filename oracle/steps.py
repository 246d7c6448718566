"""Denoising steps and the generation loop (oracle; test infrastructure only).

One object holds the whole generation state of a batch of sequences: tokens,
the per-layer K/V cache, ES-dLLM's hidden-state snapshot at the skip layer,
the latest confidence / argmax per position, SureLock's lock mask and stored
distributions, and dLLM-Cache's per-layer output cache.  `step()` runs one
denoising iteration of the configured policy:

* vanilla: every row through every layer (the full-recompute baseline).
* es: ES-dLLM summary sec. 2.1-2.2.  The first step of a block (and every
  `refresh_period` steps) recomputes all rows; other steps recompute the
  current block's rows up to the skip layer, score them by Eq. 1, keep the
  top k = ceil(keep * n) and run only those through the remaining layers.
  With `es_per_layer` the choice is made again at the start of every layer
  from the skip layer on (ES-dLLM summary sec. 2.1, item 2): Eq. 1 compares
  each candidate's input of that layer with the one of the previous
  iteration, and a row skipped at a layer carries its cached output of that
  layer (from the last iteration that computed it) into the next one.
* surelock: SureLock summary sec. 2.1.  Unlocked rows run every layer; locked
  rows are never recomputed and keep the K/V written when they locked; a row
  locks when KL(p_t || p_t-1) < eps and its confidence > tau.
* dllm_cache: dLLM-Cache explainer sec. 3.  Every `prompt_interval` steps all
  rows are recomputed; other steps recompute, per layer, only the response
  rows whose value vectors moved away from the cached ones (cosine < tau),
  at most ceil(rho * n_resp) of them.

Unmasking is top-n confidence within the current block, the DUS dilated rounds
(Plan for Speed summary sec. 2), or a confidence-bounded choice filtered by the
dilation rule (the same summary, sec. 3); a block ends when it has no masked
position left.
"""
from __future__ import annotations

import math

import numpy as np

from .model import OracleModel, lm_confidence
from .policy import (cosine_rows, dus_schedule, es_importance, kl_from_logits,
                     threshold_cap_select, topk_select, unmask_cb_dus, unmask_topconf)


class OracleRun:
    def __init__(self, cfg, weights: dict, tokens, lock_pattern=None, forced_rho: bool = False):
        self.cfg = cfg
        m = cfg.model
        self.dims = m
        self.model = OracleModel(m, weights)
        B, N = cfg.batch, cfg.seq_len
        self.B, self.N = B, N
        self.tokens = np.array(tokens, dtype=np.int64).reshape(B, N)
        L = m.n_layers
        self.K = np.zeros((L, B, m.n_kv_heads, N, m.head_dim))
        self.V = np.zeros((L, B, m.n_kv_heads, N, m.head_dim))
        self.h_prev = np.zeros((B, N, m.d_model))
        self.conf = np.zeros((B, N))
        self.amax = np.full((B, N), -1, dtype=np.int64)
        self.masked_prev = np.zeros((B, N), dtype=bool)
        self.lock = np.zeros((B, N), dtype=bool)
        self.lock_pattern = None if lock_pattern is None else np.asarray(lock_pattern, bool)
        self.prev_logits = {}          # (b, pos) -> (z, lse) of the last computed distribution
        self.forced_rho = forced_rho
        self.h_cache = None            # dLLM-Cache per-layer outputs [L, B, N, d]
        self.es_in = None              # ES per-layer: input of layer l last iteration [L, B, N, d]
        self.es_out = None             # ES per-layer: last computed output of layer l [L, B, N, d]
        self.block = 0
        self.step_in_block = 0
        self.n_steps = 0
        self.unmask_events = []        # (step, b, pos, token)
        self.last = {}                 # per-step records for tests
        if cfg.unmask == "dus":
            self.rounds = dus_schedule(cfg.block_len, cfg.dus_base)

    # ------------------------------------------------------------ helpers
    @property
    def done(self) -> bool:
        return self.block >= self.cfg.n_blocks

    def block_range(self):
        s = self.cfg.prompt_len + self.block * self.cfg.block_len
        return s, s + self.cfg.block_len

    def _rows(self, pos_lists):
        """Flatten per-sequence position lists into (b_idx, pos) arrays, b-major."""
        b_idx = np.concatenate([np.full(len(p), b, dtype=np.int64) for b, p in enumerate(pos_lists)])
        pos = np.concatenate([np.asarray(p, dtype=np.int64) for p in pos_lists])
        return b_idx, pos

    def _layers(self, h, b_idx, pos, l0, l1, keep_outputs=False):
        for l in range(l0, l1):
            if len(pos):
                h = self.model.layer(l, h, b_idx, pos, self.K[l], self.V[l])
            if keep_outputs:
                self.h_cache[l][b_idx, pos] = h
        return h

    def _lm(self, h, b_idx, pos):
        """Final norm + vocabulary projection for the given rows; stores conf/argmax."""
        if len(pos) == 0:
            return np.zeros((0, self.dims.vocab)), np.zeros(0)
        z = self.model.logits(h)
        conf, tok, lse = lm_confidence(z, self.dims.mask_id)
        self.conf[b_idx, pos] = conf
        self.amax[b_idx, pos] = tok
        return z, lse

    def _unmask(self):
        cfg = self.cfg
        s, e = self.block_range()
        committed = []
        for b in range(self.B):
            masked = self.tokens[b, s:e] == self.dims.mask_id
            if cfg.unmask == "dus":
                r = self.step_in_block
                local = [p for p in self.rounds[r] if masked[p]] if r < len(self.rounds) else \
                    [p for p in range(e - s) if masked[p]]
            elif cfg.unmask == "cb_dus":
                local = list(unmask_cb_dus(self.conf[b, s:e], masked, cfg.cb_tau, cfg.tokens_per_step))
            else:
                local = list(unmask_topconf(self.conf[b, s:e], masked, cfg.tokens_per_step))
            for p in local:
                tok = int(self.amax[b, s + p])
                self.tokens[b, s + p] = tok
                committed.append((b, s + p, tok))
                self.unmask_events.append((self.n_steps, b, s + p, tok))
        return committed

    def _advance(self):
        s, e = self.block_range()
        self.n_steps += 1
        self.step_in_block += 1
        if not np.any(self.tokens[:, s:e] == self.dims.mask_id):
            self.block += 1
            self.step_in_block = 0

    def _lm_rows_for(self, b_idx, pos, masked0):
        """Rows that need the vocabulary projection this step: computed rows that
        are masked and inside the current block (DUS: inside this round)."""
        s, e = self.block_range()
        keep = masked0[b_idx, pos] & (pos >= s) & (pos < e)
        if self.cfg.unmask == "dus" and self.step_in_block < len(self.rounds):
            in_round = np.zeros(self.N, dtype=bool)
            in_round[s + self.rounds[self.step_in_block]] = True
            keep &= in_round[pos]
        return np.nonzero(keep)[0]

    # ------------------------------------------------------------ steps
    def full_pass(self, masked0, store_hprev_rows=None, keep_outputs=False):
        """All rows through all layers (vanilla step / periodic refresh)."""
        cfg, m = self.cfg, self.dims
        b_idx, pos = self._rows([np.arange(self.N)] * self.B)
        h = self.model.embed(self.tokens[b_idx, pos])
        if keep_outputs and self.h_cache is None:
            self.h_cache = np.zeros((m.n_layers, self.B, self.N, m.d_model))
        ls = cfg.skip_layer if cfg.policy == "es" else 0
        h = self._layers(h, b_idx, pos, 0, ls, keep_outputs)
        if store_hprev_rows is not None:
            sel = store_hprev_rows[b_idx, pos]
            self.h_prev[b_idx[sel], pos[sel]] = h[sel]
        if store_hprev_rows is not None and cfg.es_per_layer:
            self._es_layer_state()
            sb, sp = b_idx[sel], pos[sel]
            for l in range(ls, m.n_layers):
                self.es_in[l][sb, sp] = h[sel]
                h = self._layers(h, b_idx, pos, l, l + 1)
                self.es_out[l][sb, sp] = h[sel]
        else:
            h = self._layers(h, b_idx, pos, ls, m.n_layers, keep_outputs)
        r = self._lm_rows_for(b_idx, pos, masked0)
        z, lse = self._lm(h[r], b_idx[r], pos[r])
        return b_idx, pos, h, r, z, lse

    def step(self, forced_scores=None):
        if self.done:
            raise RuntimeError("generation finished")
        pol = self.cfg.policy
        if pol == "vanilla":
            rec = self._vanilla_step()
        elif pol == "es":
            rec = self._es_step(forced_scores)
        elif pol == "surelock":
            rec = self._surelock_step()
        elif pol == "dllm_cache":
            rec = self._dllm_cache_step(forced_scores)
        else:
            raise ValueError(pol)
        rec["committed"] = self._unmask()
        self.last = rec
        self._advance()
        return rec

    def _vanilla_step(self):
        masked0 = self.tokens == self.dims.mask_id
        b_idx, pos, h, r, z, lse = self.full_pass(masked0)
        return {"kind": "full", "rows": (b_idx, pos), "h_out": h, "lm_rows": r}

    def _cand_positions(self):
        s, e = self.block_range()
        if self.cfg.cand_scope == "all":
            return np.arange(self.N)
        return np.arange(s, e)

    def _es_is_refresh(self) -> bool:
        rp = self.cfg.refresh_period
        return self.step_in_block == 0 or (rp > 0 and self.step_in_block % rp == 0)

    def _es_layer_state(self):
        if self.es_in is None:
            shape = (self.dims.n_layers, self.B, self.N, self.dims.d_model)
            self.es_in = np.zeros(shape)
            self.es_out = np.zeros(shape)

    def _es_step(self, forced_scores):
        cfg, m = self.cfg, self.dims
        masked0 = self.tokens == m.mask_id
        cand = self._cand_positions()
        if self._es_is_refresh():
            store = np.zeros((self.B, self.N), dtype=bool)
            store[:, cand] = True
            b_idx, pos, h, r, z, lse = self.full_pass(masked0, store_hprev_rows=store)
            self.masked_prev = masked0
            return {"kind": "refresh", "rows": (b_idx, pos), "h_out": h, "lm_rows": r}
        ls = cfg.skip_layer
        b_idx, pos = self._rows([cand] * self.B)
        h = self.model.embed(self.tokens[b_idx, pos])
        h = self._layers(h, b_idx, pos, 0, ls)
        c = np.where(self.masked_prev[b_idx, pos], self.conf[b_idx, pos], 0.0)
        if cfg.es_per_layer:
            return self._es_per_layer_skip(h, b_idx, pos, c, masked0, forced_scores)
        scores = es_importance(cfg.alpha, c, h, self.h_prev[b_idx, pos])
        self.h_prev[b_idx, pos] = h
        h_skip = h.copy()
        if forced_scores is not None:
            scores = np.asarray(forced_scores, dtype=np.float64).reshape(-1)
        n = len(cand)
        k = cfg.keep_count(n)
        act = np.concatenate([b * n + topk_select(scores[b * n:(b + 1) * n], k)
                              for b in range(self.B)])
        self.masked_prev = masked0
        ab, ap = b_idx[act], pos[act]
        ha = self._layers(h[act], ab, ap, ls, m.n_layers)
        r = self._lm_rows_for(ab, ap, masked0)
        z, lse = self._lm(ha[r], ab[r], ap[r])
        return {"kind": "skip", "rows": (ab, ap), "cand": (b_idx, pos), "scores": scores,
                "h_skip": h_skip, "active": act, "h_out": ha, "lm_rows": r, "k": k}

    def _es_per_layer_skip(self, x, b_idx, pos, c, masked0, forced_scores):
        """Layers skip_layer .. L-1 of a skip step, choosing the top k at each layer.

        x holds every candidate's input of the current layer.  forced_scores, when
        given, is one score vector per layer from the skip layer on (teacher forcing).
        """
        cfg, m = self.cfg, self.dims
        ls = cfg.skip_layer
        n = len(pos) // self.B
        k = cfg.keep_count(n)
        h_skip = x.copy()
        layer_scores, layer_active, layer_in = [], [], []
        for l in range(ls, m.n_layers):
            # Eq. 1 on this layer's input: H^(t)_l against H^(t-1)_l
            scores = es_importance(cfg.alpha, c, x, self.es_in[l][b_idx, pos])
            self.es_in[l][b_idx, pos] = x
            if forced_scores is not None:
                scores = np.asarray(forced_scores[l - ls], dtype=np.float64).reshape(-1)
            act = np.concatenate([b * n + topk_select(scores[b * n:(b + 1) * n], k)
                                  for b in range(self.B)])
            out = self.model.layer(l, x[act], b_idx[act], pos[act], self.K[l], self.V[l])
            self.es_out[l][b_idx[act], pos[act]] = out
            layer_scores.append(scores)
            layer_active.append(act)
            layer_in.append(x)
            # every candidate enters the next layer with its latest output of this one:
            # just computed for the chosen rows, cached for the skipped ones
            x = self.es_out[l][b_idx, pos].copy()
        self.masked_prev = masked0
        ab, ap = b_idx[act], pos[act]
        ha = x[act]
        r = self._lm_rows_for(ab, ap, masked0)
        self._lm(ha[r], ab[r], ap[r])
        return {"kind": "skip", "rows": (ab, ap), "cand": (b_idx, pos), "scores": layer_scores[0],
                "layer_scores": layer_scores, "layer_active": layer_active, "layer_in": layer_in,
                "h_skip": h_skip, "active": act, "h_out": ha, "lm_rows": r, "k": k}

    def _surelock_step(self):
        cfg, m = self.cfg, self.dims
        masked0 = self.tokens == m.mask_id
        lists = [np.nonzero(~self.lock[b])[0] for b in range(self.B)]
        b_idx, pos = self._rows(lists)
        h = self.model.embed(self.tokens[b_idx, pos])
        h = self._layers(h, b_idx, pos, 0, m.n_layers)
        s, e = self.block_range()
        # lock-eligible rows: the unmasked ones, or every row in the all-positions mode
        eligible = np.ones(len(pos), bool) if cfg.lock_masked else ~masked0[b_idx, pos]
        lm = eligible | (masked0[b_idx, pos] & (pos >= s) & (pos < e))
        r = np.nonzero(lm)[0]
        z = self.model.logits(h[r]) if len(r) else np.zeros((0, m.vocab))
        conf, tok, lse = (lm_confidence(z, m.mask_id) if len(r)
                          else (np.zeros(0), np.zeros(0, np.int64), np.zeros(0)))
        rb, rp = b_idx[r], pos[r]
        self.conf[rb, rp] = conf
        self.amax[rb, rp] = tok
        kl = np.full(len(r), np.nan)
        new_lock = []
        for i in range(len(r)):
            key = (int(rb[i]), int(rp[i]))
            if eligible[r[i]] and key in self.prev_logits:
                zp, lp = self.prev_logits[key]
                kl[i] = kl_from_logits(z[i:i + 1], lse[i:i + 1], zp[None], np.array([lp]))[0]
                if self.lock_pattern is not None:
                    lock_now = bool(self.lock_pattern[key])
                else:
                    lock_now = kl[i] < cfg.kl_eps and conf[i] > cfg.conf_tau
                if lock_now:
                    new_lock.append(key)
            self.prev_logits[key] = (z[i].copy(), float(lse[i]))
        for key in new_lock:
            self.lock[key] = True
        return {"kind": "surelock", "rows": (b_idx, pos), "h_out": h, "lm_rows": r,
                "kl": kl, "new_lock": new_lock, "logits": z, "lse": lse}

    def _dllm_cache_step(self, forced_scores):
        cfg, m = self.cfg, self.dims
        masked0 = self.tokens == m.mask_id
        if self.n_steps % cfg.prompt_interval == 0:
            b_idx, pos, h, r, z, lse = self.full_pass(masked0, keep_outputs=True)
            return {"kind": "refresh", "rows": (b_idx, pos), "h_out": h, "lm_rows": r}
        resp = (np.arange(self.N) if cfg.cand_scope == "all"
                else np.arange(cfg.prompt_len, self.N))
        n = len(resp)
        cap = n if cfg.rho_cap >= 1.0 else max(0, min(n, math.ceil(cfg.rho_cap * n - 1e-9)))
        b_idx, pos = self._rows([resp] * self.B)
        x = self.model.embed(self.tokens[b_idx, pos])
        per_layer = []
        for l in range(m.n_layers):
            vn = self.model.value_only(l, x)
            vc = self.V[l][b_idx, :, pos, :].reshape(len(pos), m.kv_dim)
            sims = cosine_rows(vn, vc)
            if forced_scores is not None and forced_scores[l] is not None:
                sims = np.asarray(forced_scores[l], dtype=np.float64)
            sel = np.concatenate([b * n + threshold_cap_select(sims[b * n:(b + 1) * n],
                                                               cfg.sim_tau, cap, self.forced_rho)
                                  for b in range(self.B)])
            if len(sel):
                out = self.model.layer(l, x[sel], b_idx[sel], pos[sel], self.K[l], self.V[l])
                self.h_cache[l][b_idx[sel], pos[sel]] = out
            # the next layer's input is each response row's current output of layer l
            x = self.h_cache[l][b_idx, pos].copy()
            per_layer.append({"sims": sims, "sel": sel})
        r = self._lm_rows_for(b_idx, pos, masked0)
        z, lse = self._lm(x[r], b_idx[r], pos[r])
        return {"kind": "partial", "rows": (b_idx, pos), "h_out": x, "lm_rows": r,
                "layers": per_layer}


def generate(cfg, weights, tokens, max_steps=None, **kw):
    """Run the whole generation; returns the OracleRun (tokens, events, caches)."""
    run = OracleRun(cfg, weights, tokens, **kw)
    while not run.done and (max_steps is None or run.n_steps < max_steps):
        run.step()
    return run

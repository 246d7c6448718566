#!/usr/bin/env python
"""Generated tokens/s of the token-skipping denoising generation on B200.

Workload (default): the LLaDA-8B-shaped ES-dLLM generation -- 32 layers,
d 4096, 32 heads x 128, SwiGLU 12288, vocab 126464, random-init N(0, 0.02)
bf16 weights; batch 1, a 512-token uniform-random prompt, 256 generated tokens
in blocks of 32 at 1 token per step; every block starts with a full refresh,
the other steps recompute the block's 32 rows through layers 0-3, score them
by Eq. 1 and keep the top 20% (7 rows) for layers 4-31.

One bench step = one whole generation (8 blocks x 32 denoising steps).
`value` is device-timed (CUDA events, max over ranks) with the weights and
prompt resident in HBM; `e2e` is the same generation through the public API
with the prompt copied from pinned host memory and the tokens read back each
step.  Multi-GPU runs are independent replicas (each rank generates its own
batch; the path has no exchange step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# DRAM bytes (read + write) per layer of fused_layer_kernel, from one ncu capture of the kernel on three
# LLaDA-8B-shaped layers (kernel_bench case fused_m7_l3); roofline.traffic scales it by the layers a launch runs
FUSED_DRAM_BYTES_PER_LAYER = 451.21e6
METRIC = "generated tokens/s, LLaDA-8B shape, 1×B200; step latency & roofline % vs active ratio"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return dict(PEAKS_FALLBACK, source="fallback")


def workload_desc(cfg):
    m = cfg.model
    return (f"{cfg.name}: {m.n_layers} layers, d {m.d_model}, {m.n_heads} heads x {m.head_dim} "
            f"({m.n_kv_heads} KV), SwiGLU {m.ffn_dim}, vocab {m.vocab}; batch {cfg.batch}, prompt {cfg.prompt_len}, "
            f"gen {cfg.gen_len} in blocks of {cfg.block_len}, {cfg.tokens_per_step} token/step; "
            f"ES-dLLM skip at layer {cfg.skip_layer} keeping {cfg.keep_ratio:.0%} of the block")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if uuid:
            cmd += ["-i", uuid]
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- replicas
def reduce_over_ranks(values, world: int, device="cpu"):
    """Max over ranks of each per-rank value (device times, wall times); with one rank the
    values are returned unchanged.  Replicas exchange nothing else: each rank generates its
    own batch, so whole-job throughput = tokens of all ranks / the slowest rank's time."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tokens_per_s(batch: int, gen_len: int, steps: int, world: int, seconds: float) -> float:
    return batch * gen_len * steps * world / seconds


def step_work(m, rows_per_layer, lm_rows, N, batch):
    """Algorithmic bytes and FLOPs of one denoising step: every layer streams its weights
    (2 P bytes) and reads its K/V cache, the recomputed rows of each layer do 2 P FLOPs of
    GEMM and 4 N Hq hd of attention, the vocabulary projection streams V d weights."""
    P = m.params_per_layer
    byts = sum(2.0 * P + 2.0 * batch * N * m.kv_dim * 2 + r * (2 * m.kv_dim + 2 * m.d_model) * 2
               for r in rows_per_layer) + 2.0 * m.vocab * m.d_model
    flops = sum(2.0 * r * P + 4.0 * r * N * m.n_heads * m.head_dim for r in rows_per_layer)
    flops += 2.0 * lm_rows * m.vocab * m.d_model
    return byts, flops


def generation_roofline(cfg, peaks, measured_ms):
    """Roofline of one whole ES-dLLM generation: each step is bound by its bytes at the measured
    HBM bandwidth or its FLOPs at the sustained bf16 peak (the generation is a long loop),
    whichever is slower; refresh steps recompute every row, skip steps the block's rows below
    the skip layer and the kept rows above it."""
    m, N, B = cfg.model, cfg.seq_len, cfg.batch
    L, ls, n_c = m.n_layers, cfg.skip_layer, cfg.block_len
    k = cfg.keep_count(n_c)
    steps_per_block = math.ceil(cfg.block_len / cfg.tokens_per_step)
    n_ref = cfg.n_blocks
    n_skip = cfg.n_blocks * (steps_per_block - 1)
    hbm, tc = peaks["hbm_gbs"] * 1e6, peaks["bf16_tflops_sustained"] * 1e9        # bytes / ms, flops / ms
    b_s, f_s = step_work(m, [B * n_c] * ls + [B * k] * (L - ls), B * k, N, B)
    b_r, f_r = step_work(m, [B * N] * L, B * n_c, N, B)
    t_s, t_r = max(b_s / hbm, f_s / tc), max(b_r / hbm, f_r / tc)
    roof_ms = n_ref * t_r + n_skip * t_s
    return {"roofline_ms": round(roof_ms, 2), "measured_ms": round(measured_ms, 2),
            "frac": round(roof_ms / measured_ms, 4),
            "tokens_per_s_at_roofline": round(B * cfg.gen_len / (roof_ms / 1e3), 2),
            "skip_step": {"count": n_skip, "roofline_ms": round(t_s, 4), "bound": "hbm" if b_s / hbm >= f_s / tc else "tensor",
                          "bytes": round(b_s), "flops": round(f_s)},
            "refresh_step": {"count": n_ref, "roofline_ms": round(t_r, 4),
                             "bound": "hbm" if b_r / hbm >= f_r / tc else "tensor", "bytes": round(b_r), "flops": round(f_r)},
            "peaks": f"HBM {peaks['hbm_gbs']} GB/s, bf16 {peaks['bf16_tflops_sustained']} TFLOP/s sustained "
                     f"({peaks['source']})"}


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from synth import get_config, make_tokens, make_weights
    from synth.gen import PROMPT_SEED
    from token_skip_denoising_b200.engine import Engine, kernel_launches

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = get_config(args.workload)
    peaks = load_peaks()
    w = make_weights(cfg.model, device=dev)
    tok0_host = make_tokens(cfg, seed=PROMPT_SEED + rank).pin_memory()
    tok0 = tok0_host.to(dev)
    tok = tok0.clone()
    stream = torch.cuda.current_stream(dev)
    eng = Engine(cfg, w, tok, stream=stream)

    def one_generation():
        eng.reset(tok0)
        eng.generate()

    for _ in range(args.warmup):
        one_generation()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- device-timed region: K generations, nothing else on the stream
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(uuid)
    launches0 = kernel_launches()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        one_generation()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = kernel_launches() - launches0
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    ms_max = reduce_over_ranks([ms], world, dev)[0]
    value = whole_job_tokens_per_s(cfg.batch, cfg.gen_len, args.steps, world, ms_max / 1e3)
    assert not bool((tok == cfg.model.mask_id).any()), "generation left mask ids"

    # ---- end to end through the public API, host buffers, copies inside the region
    out_host = torch.empty_like(tok0_host).pin_memory()
    barrier()
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    for _ in range(args.steps):
        tok.copy_(tok0_host, non_blocking=True)      # H2D of this step's input
        eng.reset()
        eng.generate()
        out_host.copy_(tok, non_blocking=True)       # D2H of the result
    torch.cuda.synchronize()
    e2e_s = reduce_over_ranks([time.perf_counter() - w0], world, dev)[0]
    e2e_value = whole_job_tokens_per_s(cfg.batch, cfg.gen_len, args.steps, world, e2e_s)

    # ---- per-kernel figures: one more generation with every launch bracketed by CUDA events
    # (on the engine's stream); the dominant kernel is the fused run of layers of the skip steps
    eng.profile(1, peaks["hbm_gbs"], peaks["bf16_tflops_sustained"])
    eng.profile_read()
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    one_generation()
    p1.record(stream)
    torch.cuda.synchronize()
    prof = eng.profile_read()
    eng.profile(0)
    prof_ms = p0.elapsed_time(p1)
    fused_gbs = prof["fused_bytes"] / (prof["fused_ms"] / 1e3) / 1e9 if prof["fused_ms"] > 0 else 0.0
    layers_per_launch = prof["fused_layers"] / max(1, prof["fused_launches"])
    roof = {"bound": "hbm", "achieved": round(fused_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(fused_gbs / peaks["hbm_gbs"], 4),
            "traffic": round(FUSED_DRAM_BYTES_PER_LAYER * layers_per_launch),
            "traffic_source": "ncu dram read+write of one 3-layer launch (7 rows), per layer, x layers per launch",
            "kernel": "fused_layer_kernel (one persistent launch per run of layers with <= 64 rows)",
            "peak_source": peaks["source"],
            "launches": prof["fused_launches"], "layers_per_launch": round(layers_per_launch, 2),
            "avg_launch_us": round(1e3 * prof["fused_ms"] / max(1, prof["fused_launches"]), 2),
            "bytes_per_launch": round(prof["fused_bytes"] / max(1, prof["fused_launches"])),
            "time_share": round(prof["fused_ms"] / prof_ms, 4) if prof_ms else None,
            "timing": "every launch of one extra generation bracketed by CUDA events on the engine stream",
            "split_path": {"kernel": "gemm_tc_kernel + attn_kernel (rows > 64: refresh steps)",
                           "gemm_launches": prof["gemm_launches"],
                           "gemm_time_share": round(prof["gemm_ms"] / prof_ms, 4) if prof_ms else None,
                           "gemm_achieved_tflops": round(prof["gemm_flops"] / (prof["gemm_ms"] / 1e3) / 1e12, 1)
                           if prof["gemm_ms"] else None,
                           "gemm_roofline_time_frac": round(prof["gemm_roofline_ms"] / prof["gemm_ms"], 4)
                           if prof["gemm_ms"] else None,
                           "attn_time_share": round(prof["attn_ms"] / prof_ms, 4) if prof_ms else None}}
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded random-init N(0,0.02) bf16 weights, uniform-random prompt ids",
        "config": {"workload": workload_desc(cfg), "batch": cfg.batch, "seq_len": cfg.seq_len,
                   "gen_len": cfg.gen_len, "step": "one whole generation (all blocks and denoising steps)",
                   "l2": "inputs larger than L2: every denoising step streams all 16 GB of weights",
                   "parallelism": f"replicas x{world} (no collective)"},
        "roofline": roof,
        "generation_roofline": generation_roofline(cfg, peaks, ms_max / args.steps),
        "e2e": {"value": round(e2e_value, 3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(tok0_host.numel() * 4), "d2h_bytes_per_step": int(out_host.numel() * 4)},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    return line, eng, w, cfg


# ---------------------------------------------------------------- active-ratio sweep (single layer)
def micro_sweep(peaks, reps=20):
    """Single-layer step at N = 2048 (d 4096, 32 heads, FFN 12288): score -> top-k ->
    gathered QKV/O/FFN -> active-query attention -> K/V scatter, for each active ratio; the
    step's launches replay as one CUDA graph after an L2 flush."""
    import torch

    from synth import get_config, make_weights
    from synth.gen import kv_cache_fill, microbench_active, microbench_hidden
    from token_skip_denoising_b200 import _lib, ops

    cfg = get_config("micro")
    m = cfg.model
    N, d = cfg.seq_len, m.d_model
    w = make_weights(m, device="cuda")
    lw = {k: w[k][0] for k in ("w_qkv", "w_o", "w_gu", "w_down", "g_attn", "g_ffn")}
    kv = kv_cache_fill(1, 1, m.n_kv_heads, N, m.head_dim, device="cuda")
    kc, vc = kv[0, 0].contiguous(), kv[0, 1].contiguous()
    hin = microbench_hidden(N, d, device="cuda")
    cos, sin = ops.rope_table(N, m.head_dim, m.rope_theta)
    ccfg = _lib.make_config(cfg)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    out = []
    P = m.params_per_layer
    # the oracle's single-layer step on the host: Eq. 1 over the N rows, the top k, the layer on
    # the k rows (measured up to 512 rows, scaled by rows beyond: labelled extrapolated)
    from oracle.policy import es_importance, topk_select
    lw_host = layer_weights_cpu(w, 0)
    h_host, hp_host = hin["h_cur"].double().cpu().numpy(), hin["h_prev"].double().cpu().numpy()
    c_host = hin["conf"].double().cpu().numpy() * hin["masked_prev"].cpu().numpy()
    rng = np.random.default_rng(0)
    cores = host_cores()
    for rho in (0.03, 0.1, 0.25, 0.5, 1.0):
        k = max(1, math.ceil(rho * N - 1e-9))
        t = time.perf_counter()
        topk_select(es_importance(0.5, c_host, h_host, hp_host), k)
        o_ms = 1e3 * (time.perf_counter() - t + oracle_layer_s(m, lw_host, k, N, rng, cap=512))
        oracle = {"ms": round(o_ms, 1), "cores": cores, "kind": "oracle",
                  "sample": "fp64 oracle: Eq. 1, top k, one layer" + (f" (layer measured at 512 rows, scaled x{k / 512:.2f}:"
                                                                     " extrapolated)" if k > 512 else "")}
        ws = torch.zeros(ops.layer_workspace_bytes(ccfg, k, k), dtype=torch.uint8, device="cuda")
        for pattern in ("random", "contiguous"):
            h = hin["h_cur"].clone()
            hp = hin["h_prev"].clone()
            act_idx = microbench_active(N, k, pattern).cuda()
            cnt = torch.tensor([k], dtype=torch.int32, device="cuda")
            off = torch.tensor([0, k], dtype=torch.int32, device="cuda")
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

            def step():
                s = ops.score_es(h, hp, hin["conf"], 0.5, masked_prev=hin["masked_prev"])
                ops.select(s, 1, N, ops.SEL_TOPK_DESC, k)
                # the layer runs on the fixed index pattern so both patterns are measured
                ops.layer(ccfg, lw, kc, vc, cos, sin, h, act_idx, cnt, off, k, k, ws=ws)

            # the three launches replay as one CUDA graph, so the host's per-call marshalling
            # does not pace the GPU (at 62 rows it would add ~100 us of idle device time)
            step()
            torch.cuda.synchronize()
            cs = torch.cuda.Stream()
            cs.wait_stream(torch.cuda.current_stream())
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.stream(cs):
                with torch.cuda.graph(graph, stream=cs):
                    step()
            torch.cuda.synchronize()
            times = []
            for it in range(reps + 3):
                flush.zero_()
                ev[0].record()
                graph.replay()
                ev[1].record()
                torch.cuda.synchronize()
                if it >= 3:
                    times.append(ev[0].elapsed_time(ev[1]))
            del graph
            t = statistics.median(times)
            kv_bytes = 2 * N * m.kv_dim * 2
            byts = P * 2 + kv_bytes + k * (2 * m.kv_dim + 2 * d) * 2 + 2 * N * d * 4
            flops = 2 * k * P + 4 * k * N * m.n_heads * m.head_dim
            roof_ms = max(byts / (peaks["hbm_gbs"] * 1e6), flops / (peaks["bf16_tflops"] * 1e9))
            out.append({"rho": rho, "k": k, "pattern": pattern, "ms": round(t, 4),
                        "roofline_ms": round(roof_ms, 4), "roofline_frac": round(roof_ms / t, 4),
                        "cpu_baseline": oracle,
                        "bound": "hbm" if byts / (peaks["hbm_gbs"] * 1e6) >= flops / (peaks["bf16_tflops"] * 1e9)
                        else "tensor"})
    del w
    return out


# ---------------------------------------------------------------- SureLock / dLLM-Cache steps
def _timed_steps(eng, n, stream):
    """Device time (ms) of each of the next n denoising steps, one event pair per step."""
    import torch
    out = []
    for _ in range(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        eng.step()
        e1.record(stream)
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1))
    return out


def _step_roofline_ms(peaks, m, n_layers_rows, lm_rows, N, batch, extra_bytes=0.0):
    """max(weight + K/V + extra bytes at HBM bandwidth, active-row FLOPs at the sustained
    bf16 peak) for one step; n_layers_rows = the active row count of each layer."""
    P = m.params_per_layer
    flops = sum(2.0 * r * P + 4.0 * r * N * m.n_heads * m.head_dim for r in n_layers_rows)
    flops += 2.0 * lm_rows * m.vocab * m.d_model
    byts = len(n_layers_rows) * (2.0 * P + 2.0 * batch * N * m.kv_dim * 2) + 2.0 * m.vocab * m.d_model
    byts += extra_bytes
    t_b = byts / (peaks["hbm_gbs"] * 1e6)
    t_f = flops / (peaks["bf16_tflops_sustained"] * 1e9)
    return max(t_b, t_f), ("hbm" if t_b >= t_f else "tensor")


def variant_steps(peaks, steps=3, warm=2):
    """Per-step device latency of the SureLock (Dream-7B shape, batch 8) and dLLM-Cache + DUS
    (long-context LLaDA-8B shape, batch 4) generations, at the measured selection and at
    forced lock fractions / a forced cap, with tokens/s extrapolated to a whole run; and whole
    LLaDA-8B ES-dLLM generations with several tokens per step (top-n confidence, and the
    confidence-bounded sampler filtered by the DUS dilation rule)."""
    import numpy as np
    import torch

    from synth import get_config, lock_pattern, make_tokens, make_weights
    from token_skip_denoising_b200.engine import Engine

    stream = torch.cuda.current_stream()
    res = {}
    # ---- SureLock, Dream-7B shape
    cfg = get_config("dream_surelock")
    m, B, N = cfg.model, cfg.batch, cfg.seq_len
    w = make_weights(m, device="cuda")
    tok0 = make_tokens(cfg).cuda()
    eng = Engine(cfg, w, tok0.clone(), stream=stream)
    rows = []
    rng = np.random.default_rng(0)
    lw_host = layer_weights_cpu(w, 0)
    lm_host, gf_host = w["lm_head"].cpu(), w["g_final"].cpu()
    cores = host_cores()
    # oracle seconds per layer (weight conversion) and per active row of a layer (a 256-row sample),
    # per vocabulary-projection row (a 64-row sample)
    o_conv, o_row = oracle_layer_cost(m, lw_host, 256, N, rng)
    o_lm_row = oracle_lm_s(m, lm_host, gf_host, 64, rng) / 64
    for frac in (None, 0.25, 0.5, 0.75):
        eng.reset(tok0)
        pat = lock_pattern(B, N, frac).cuda() if frac is not None else None
        eng.set_lock_pattern(pat)
        _timed_steps(eng, warm, stream)                # step 0 computes every row; step 1 locks
        t = statistics.median(_timed_steps(eng, steps, stream))
        locked = int(eng.buffer("lock").sum())
        active = int(eng.buffer("nrows")[0])
        n_lm = int(eng.buffer("nlmrows")[0])
        # logits of the recomputed rows: one store, three reads of this step's, one of the previous
        logit_bytes = 5.0 * n_lm * m.vocab * 2
        roof, bound = _step_roofline_ms(peaks, m, [active] * m.n_layers, n_lm, N, B, logit_bytes)
        o_ms = 1e3 * (m.n_layers * (o_conv + active * o_row) + n_lm * o_lm_row)
        rows.append({"lock": "rule (KL < eps and conf > tau)" if frac is None else f"forced {frac:.2f} of positions",
                     "locked_frac": round(locked / (B * N), 4), "active_rows": active, "lm_rows": n_lm,
                     "ms_per_step": round(t, 3), "tokens_per_s": round(B * cfg.tokens_per_step / (t / 1e3), 2),
                     "roofline_ms": round(roof, 3), "roofline_frac": round(roof / t, 4), "bound": bound,
                     "cpu_baseline": {"ms_per_step": round(o_ms, 1), "cores": cores, "kind": "oracle",
                                      "sample": "fp64 oracle, one layer at 256 rows and the vocabulary projection "
                                                "of 64 rows, scaled to the step's rows and layers: extrapolated"}})
    eng.set_lock_pattern(None)
    res["surelock_dream7b_b8"] = {
        "workload": f"{cfg.name}: batch {B}, prompt {cfg.prompt_len}, gen {cfg.gen_len} in blocks of "
                    f"{cfg.block_len}, 1 token/step; lock when KL < {cfg.kl_eps} and conf > {cfg.conf_tau}",
        "tokens_per_s": "per step: batch x tokens per step / step time (the lock fraction of that step)",
        "cases": rows}
    del eng
    w.clear()
    torch.cuda.empty_cache()

    # ---- dLLM-Cache + DUS, long-context LLaDA-8B shape
    cfg = get_config("llada_cache_dus")
    m, B, N = cfg.model, cfg.batch, cfg.seq_len
    w = make_weights(m, device="cuda")
    tok0 = make_tokens(cfg).cuda()
    n_resp = B * cfg.gen_len
    rng = np.random.default_rng(0)
    lw_host = layer_weights_cpu(w, 0)
    o_conv, o_row = oracle_layer_cost(m, lw_host, 256, N, rng)
    o_lm_row = oracle_lm_s(m, w["lm_head"].cpu(), w["g_final"].cpu(), 64, rng) / 64
    from oracle.model import OracleModel
    hv = rng.standard_normal((256, m.d_model))
    om_v = OracleModel(m, lw_host)
    t = time.perf_counter()
    om_v.value_only(0, hv)
    o_probe_row = (time.perf_counter() - t) / 256          # the value-vector probe of one response row
    cores = host_cores()
    R = max(1, math.ceil(math.log2(cfg.block_len)))
    n_steps = cfg.n_blocks * R
    n_ref = math.ceil(n_steps / cfg.prompt_interval)
    rows = []
    for forced in (0, 1):
        eng = Engine(cfg, w, tok0.clone(), stream=stream, forced_rho=forced)
        t_full = _timed_steps(eng, 1, stream)[0]               # step 0: full refresh
        _timed_steps(eng, warm, stream)
        t_part = statistics.median(_timed_steps(eng, steps, stream))
        # selected rows of every layer, from one more (untimed) step taken layer by layer
        eng.begin_step()
        sel = []
        for layer in range(m.n_layers):
            eng.layer_forward(layer)
            sel.append(int(eng.buffer("nsel")[0]))
        eng.unmask()
        torch.cuda.synchronize()
        lm_rows = int(eng.buffer("nlmrows")[0])
        hid_bytes = m.n_layers * 2.0 * n_resp * m.d_model * 4          # cached layer inputs and outputs
        roof_p, bound_p = _step_roofline_ms(peaks, m, sel, lm_rows, N, B, hid_bytes)
        vproj = m.n_layers * 2.0 * n_resp * m.d_model * m.kv_dim / (peaks["bf16_tflops_sustained"] * 1e9)
        roof_p = max(roof_p, vproj)
        roof_f, _ = _step_roofline_ms(peaks, m, [B * N] * m.n_layers, lm_rows, N, B)
        gen_s = (n_ref * t_full + (n_steps - n_ref) * t_part) / 1e3
        o_part = 1e3 * (m.n_layers * o_conv + sum(sel) * o_row + m.n_layers * n_resp * o_probe_row + lm_rows * o_lm_row)
        o_full = 1e3 * (m.n_layers * (o_conv + B * N * o_row) + lm_rows * o_lm_row)
        rows.append({"cpu_baseline": {"partial_ms": round(o_part, 1), "refresh_ms": round(o_full, 1), "cores": cores,
                                      "kind": "oracle",
                                      "sample": "fp64 oracle, one layer at 256 rows, the value probe of 256 rows and "
                                                "the vocabulary projection of 64 rows, scaled to the step's rows and "
                                                "layers: extrapolated"},
                     "selection": "forced: exactly the cap" if forced else f"cos < {cfg.sim_tau}, capped",
                     "rho_mean": round(float(np.mean(sel)) / n_resp, 4), "sel_rows_per_layer_max": max(sel),
                     "refresh_ms": round(t_full, 3), "partial_ms": round(t_part, 3),
                     "partial_roofline_ms": round(roof_p, 3), "partial_roofline_frac": round(roof_p / t_part, 4),
                     "partial_bound": bound_p,
                     "refresh_roofline_ms": round(roof_f, 3), "refresh_roofline_frac": round(roof_f / t_full, 4),
                     "tokens_per_s": round(B * cfg.gen_len / gen_s, 2)})
        del eng
        torch.cuda.empty_cache()
    # ---- ES-dLLM with parallel decoding (several top-confidence tokens per step), same weights
    es = get_config("llada_es")
    es_rows = []
    for n in (2, 4):
        ecfg = es.replace(tokens_per_step=n)
        etok = make_tokens(ecfg).cuda()
        eng = Engine(ecfg, w, etok.clone(), stream=stream)
        eng.generate()                                          # warm-up generation
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        eng.reset(etok)
        torch.cuda.synchronize()
        e0.record(stream)
        eng.generate()
        e1.record(stream)
        torch.cuda.synchronize()
        gen_ms = e0.elapsed_time(e1)
        steps = ecfg.n_blocks * math.ceil(ecfg.block_len / n)
        es_rows.append({"tokens_per_step": n, "steps": steps, "generation_ms": round(gen_ms, 2),
                     "tokens_per_s": round(ecfg.batch * ecfg.gen_len / (gen_ms / 1e3), 2)})
        del eng
        torch.cuda.empty_cache()
    res["es_parallel_decoding_llada8b"] = {
        "workload": "llada_es with n top-confidence tokens committed per step (one generation, device-timed)",
        "cases": es_rows}
    # ---- ES-dLLM with the top k chosen again at every layer from the skip layer on
    ecfg = es.replace(es_per_layer=True)
    etok = make_tokens(ecfg).cuda()
    eng = Engine(ecfg, w, etok.clone(), stream=stream)
    eng.generate()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    eng.reset(etok)
    torch.cuda.synchronize()
    e0.record(stream)
    eng.generate()
    e1.record(stream)
    torch.cuda.synchronize()
    gen_ms = e0.elapsed_time(e1)
    res["es_per_layer_llada8b"] = {
        "workload": "llada_es with the top k re-chosen by Eq. 1 at every layer from the skip layer on "
                    "(skip steps: layers 4-31 in one persistent launch that scores and chooses the rows at the "
                    "start of each layer; one generation, device-timed)",
        "generation_ms": round(gen_ms, 2), "steps": ecfg.n_blocks * ecfg.block_len,
        "tokens_per_s": round(ecfg.batch * ecfg.gen_len / (gen_ms / 1e3), 2)}
    del eng
    torch.cuda.empty_cache()
    # ---- ES-dLLM with confidence-bounded unmasking filtered by the DUS dilation rule; random
    # weights give every token a confidence near 1/V, so the bound is set to 0 and the cap and the
    # non-adjacency rule decide how many tokens a step takes
    es_rows = []
    for n in (2, 4, 8):
        ecfg = es.replace(unmask="cb_dus", cb_tau=0.0, tokens_per_step=n)
        etok = make_tokens(ecfg).cuda()
        eng = Engine(ecfg, w, etok.clone(), stream=stream)
        eng.generate()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        eng.reset(etok)
        torch.cuda.synchronize()
        gen_steps = 0
        e0.record(stream)
        while not eng.done:
            eng.step()
            gen_steps += 1
        e1.record(stream)
        torch.cuda.synchronize()
        gen_ms = e0.elapsed_time(e1)
        es_rows.append({"cap": n, "steps": gen_steps, "generation_ms": round(gen_ms, 2),
                     "tokens_per_s": round(ecfg.batch * ecfg.gen_len / (gen_ms / 1e3), 2)})
        del eng
        torch.cuda.empty_cache()
    res["es_cb_dus_llada8b"] = {
        "workload": "llada_es, unmask = confidence-bounded (tau 0) with the dilation post-filter, cap n per step; "
                    "each step syncs the host once (data-dependent block ends)",
        "cases": es_rows}
    res["dllm_cache_dus_llada8b_b4"] = {
        "workload": f"{cfg.name}: batch {B}, prompt {cfg.prompt_len}, gen {cfg.gen_len} in blocks of "
                    f"{cfg.block_len}, DUS {R} rounds/block; prompt refresh every {cfg.prompt_interval} steps; "
                    f"cos < {cfg.sim_tau} capped at rho {cfg.rho_cap}",
        "tokens_per_s": f"{n_ref} refresh + {n_steps - n_ref} partial steps at the measured step times",
        "cases": rows}
    w.clear()
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- oracle timing (CPU)
def host_cores():
    try:
        from threadpoolctl import threadpool_info
        return int(max([i.get("num_threads", 1) for i in threadpool_info()] + [1]))
    except Exception:
        return int(os.cpu_count() or 1)


def layer_weights_cpu(w, layer):
    """One layer of a weight dict (device or host tensors) as the oracle's host weights."""
    lw = {key: w[key][layer:layer + 1].cpu() for key in ("w_qkv", "w_o", "w_gu", "w_down", "g_attn", "g_ffn")}
    lw["layers"] = [0]
    return lw


def oracle_layer_cost(m, lw, r, N, rng):
    """(seconds of the fp64 oracle's weight conversion for one layer, seconds per row of the layer
    itself) from one layer on r rows of one sequence of N positions: every layer of an oracle step
    converts its weights once, and the rest of its work is linear in its rows."""
    from oracle.model import OracleModel
    om = OracleModel(m, lw)
    K = np.zeros((1, m.n_kv_heads, N, m.head_dim))
    V = np.zeros_like(K)
    h = rng.standard_normal((r, m.d_model))
    pos = np.sort(rng.choice(N, r, replace=False))
    t = time.perf_counter()
    om.layer_weights(0)
    t_conv = time.perf_counter() - t
    t = time.perf_counter()
    om.layer(0, h, np.zeros(r, dtype=np.int64), pos, K, V)
    return t_conv, (time.perf_counter() - t) / r


def oracle_layer_s(m, lw, rows, N, rng, cap=None):
    """Host seconds of one fp64 oracle layer on `rows` rows, its weight conversion included; with a
    cap, the rows' part is measured at `cap` rows and scaled by rows / cap."""
    r = rows if cap is None else min(rows, cap)
    t_conv, t_row = oracle_layer_cost(m, lw, r, N, rng)
    return t_conv + t_row * rows


def oracle_lm_s(m, lm_head, g_final, rows, rng, cap=None):
    """Host seconds of the oracle's final RMSNorm + vocabulary projection + confidence of `rows`
    rows (scaled from `cap` rows when capped)."""
    from oracle.model import OracleModel, lm_confidence
    r = rows if cap is None else min(rows, cap)
    om = OracleModel(m, {"lm_head": lm_head, "g_final": g_final, "layers": []})
    h = rng.standard_normal((r, m.d_model))
    t = time.perf_counter()
    lm_confidence(om.logits(h), m.mask_id)
    return (time.perf_counter() - t) * rows / r


def oracle_generation_sample(cfg, layers_w, lm_head, g_final, rng):
    """One bounded sample of an ES-dLLM generation on the oracle: one layer at each row count a
    generation uses (every row at a refresh, the block below the skip layer, the kept rows above
    it) and the vocabulary projection of the block's rows at a refresh and of the kept rows at a
    skip step.  Returns (generation seconds extrapolated to every step and layer, sample seconds)."""
    m = cfg.model
    N, n_c = cfg.seq_len, cfg.block_len
    k = cfg.keep_count(n_c)
    B = cfg.batch
    t0 = time.perf_counter()
    t_full = oracle_layer_s(m, layers_w[0], N, N, rng)
    t_pre = oracle_layer_s(m, layers_w[1], n_c, N, rng)
    t_post = oracle_layer_s(m, layers_w[2], k, N, rng)
    t_lm_ref = oracle_lm_s(m, lm_head, g_final, n_c, rng)
    t_lm = oracle_lm_s(m, lm_head, g_final, k, rng)
    spent = time.perf_counter() - t0
    steps_per_block = math.ceil(cfg.block_len / cfg.tokens_per_step)
    n_ref, n_skip = cfg.n_blocks, cfg.n_blocks * (steps_per_block - 1)
    L, ls = m.n_layers, cfg.skip_layer
    gen_s = B * (n_ref * (L * t_full + t_lm_ref) + n_skip * (ls * t_pre + (L - ls) * t_post + t_lm))
    return gen_s, spent


def generation_sample_desc(cfg):
    m = cfg.model
    k = cfg.keep_count(cfg.block_len)
    steps_per_block = math.ceil(cfg.block_len / cfg.tokens_per_step)
    return (f"fp64 oracle, per sample: one layer at {cfg.seq_len}, {cfg.block_len} and {k} rows and the "
            f"vocabulary projection of {cfg.block_len} and {k} rows (weight conversion included), extrapolated "
            f"to {cfg.n_blocks} refresh + {cfg.n_blocks * (steps_per_block - 1)} skip steps of {m.n_layers} layers")


def oracle_sample_timing(cfg, w_dev):
    """cpu_baseline of our arm: the oracle on one sample of the generation (host cores)."""
    rng = np.random.default_rng(0)
    layers_w = [layer_weights_cpu(w_dev, l) for l in range(3)]
    gen_s, spent = oracle_generation_sample(cfg, layers_w, w_dev["lm_head"].cpu(), w_dev["g_final"].cpu(), rng)
    return {"value": round(cfg.batch * cfg.gen_len / gen_s, 6), "unit": "tokens/s", "cores": host_cores(),
            "kind": "oracle", "sample": generation_sample_desc(cfg) + f" ({spent:.1f} s of host time)"}


# ---------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    from synth import get_config
    from synth.gen import make_weights

    cfg = get_config(args.workload)
    m = cfg.model
    # host weights of the three sampled layers and the vocabulary, seeded like the GPU arm's draw
    w = make_weights(m, device="cpu", layers=[0, 1, 2])
    layers_w = [layer_weights_cpu(w, i) for i in range(3)]
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        oracle_generation_sample(cfg, layers_w, w["lm_head"], w["g_final"], rng)
    gens, samples = [], []
    for _ in range(args.steps):
        g, sp = oracle_generation_sample(cfg, layers_w, w["lm_head"], w["g_final"], rng)
        gens.append(g)
        samples.append(sp)
    value = cfg.batch * cfg.gen_len * args.steps / sum(gens)
    desc = generation_sample_desc(cfg)
    line = {"metric": METRIC, "value": round(value, 6), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * sum(samples) / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "impl": "reference",
            "data": "synthetic: seeded random-init N(0,0.02) bf16 weights, uniform-random prompt ids",
            "config": {"workload": workload_desc(cfg), "batch": cfg.batch, "seq_len": cfg.seq_len,
                       "gen_len": cfg.gen_len,
                       "step": "one bounded sample of the generation (ms_per_step is its host time); value is the "
                               "generation's tokens/s extrapolated from the samples",
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 6), "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llada_es")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3          # timing rule: at least three untimed warm-up steps

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    line, eng, w, cfg = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1:
        peaks = load_peaks()
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_sample_timing(cfg, w)
        del eng
        if not args.no_sweep:
            w.clear()
            torch.cuda.empty_cache()
            line["active_ratio_sweep"] = micro_sweep(peaks)
        if not args.no_variants:
            w.clear()
            torch.cuda.empty_cache()
            line["variant_steps"] = variant_steps(peaks)
    elif rank == 0:
        line["cpu_baseline"] = None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

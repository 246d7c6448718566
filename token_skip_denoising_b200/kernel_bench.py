"""Kernel-level microbenchmark of the CUDA path (also the target of ncu captures).

    python -m token_skip_denoising_b200.kernel_bench [--case NAME] [--reps R] [--json]

Cases time one kernel family at the LLaDA-8B shape on seeded inputs: the fused
GEMM of each projection at the active-row counts of a skip step (7, 32) and of a
refresh (768), the attention of the active rows over N = 768 cached keys, the
LM head, and the persistent run of layers of a skip step (7 or 32 rows over a
few LLaDA-8B-shaped layers, through the engine).  Each weight matrix is replicated enough times that the working
set exceeds L2 (126 MB) and the copies are used round-robin, so the timings
are HBM timings.  Durations are CUDA-event medians; bytes and flops are the
algorithmic ones (weights + activation rows + outputs).
"""
from __future__ import annotations

import argparse
import json
import math
import statistics

import torch

from . import ops

L2_BYTES = 126 << 20


def _copies(nbytes):
    return max(2, math.ceil(3 * L2_BYTES / nbytes))


def _time(fn, reps, warm=3):
    """Per-call device time: `reps` calls are captured in one CUDA graph and the
    graph replay is timed, so host-side argument marshalling does not pace the GPU."""
    for i in range(warm):
        fn(i)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(reps):
                fn(warm + i)
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) / reps)
    return statistics.median(times)


def gemm_case(kind, rows, reps, d=4096, F=12288, V=126464, splits=0, bn=0):
    g = torch.Generator(device="cuda").manual_seed(0)
    shapes = {"qkv": (3 * d, d), "o": (d, d), "gu": (2 * F, d), "down": (d, F), "lm": (V, d)}
    n_out, K = shapes[kind]
    nbytes = n_out * K * 2
    ncop = _copies(nbytes) if kind != "lm" else 1
    Ws = [(torch.randn((n_out, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16) for _ in range(ncop)]
    X = torch.randn((rows, K), generator=g, device="cuda").to(torch.bfloat16)
    ws = torch.zeros(256 << 20, dtype=torch.uint8, device="cuda")
    out_bytes = rows * n_out * 4
    if kind == "gu":
        fn = lambda i: ops.gate_up(Ws[i % ncop], X, F, splits=splits, ws=ws)
        out_bytes = rows * F * 2
    elif kind == "lm":
        wsl = torch.zeros(max(256 << 20, rows * (V // 128) * 16 + (64 << 20)), dtype=torch.uint8, device="cuda")
        fn = lambda i: ops.lm_head(Ws[0], X, V - 1, ws=wsl)
        out_bytes = rows * (V // 128) * 16
    else:
        out = torch.empty((rows, n_out), dtype=torch.float32, device="cuda")
        fn = lambda i: ops.gemm(Ws[i % ncop], X, kind=0, out=out, splits=splits, bn=bn, ws=ws)
    t = _time(fn, reps)
    byts = nbytes + rows * K * 2 + out_bytes
    flops = 2.0 * rows * n_out * K
    return {"case": f"gemm_{kind}_m{rows}", "ms": t, "gbs": byts / t / 1e6, "tflops": flops / t / 1e9,
            "bytes": byts, "flops": flops}


def attn_case(rows, reps, N=768, H=32, hd=128, splits=0):
    from synth.configs import LLADA8B
    g = torch.Generator(device="cuda").manual_seed(1)
    kvb = 2 * H * N * hd * 2
    ncop = _copies(kvb)
    caches = [(torch.randn((1, H, N, hd), generator=g, device="cuda").to(torch.bfloat16),
               torch.randn((1, H, N, hd), generator=g, device="cuda").to(torch.bfloat16)) for _ in range(ncop)]
    q = torch.randn((rows, H * hd), generator=g, device="cuda").to(torch.bfloat16)
    off = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
    ws = torch.zeros(256 << 20, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    fn = lambda i: ops.attention(q, caches[i % ncop][0], caches[i % ncop][1], off, LLADA8B, rows, splits=splits,
                                 out=out, ws=ws)
    t = _time(fn, reps)
    byts = kvb + 2 * rows * H * hd * 2
    flops = 4.0 * rows * N * H * hd
    return {"case": f"attn_m{rows}_n{N}", "ms": t, "gbs": byts / t / 1e6, "tflops": flops / t / 1e9,
            "bytes": byts, "flops": flops}


def fused_case(rows, reps, layers=3):
    """A skip step's run of `layers` layers as one persistent kernel (7 kept or 32 candidate rows)."""
    from synth import get_config, make_tokens, make_weights
    from synth.configs import scaled
    from .engine import Engine
    base = scaled(get_config("llada_es"), n_layers=layers + 1, vocab=2048, mask_id=2047)
    cfg = base.replace(skip_layer=1) if rows < base.block_len else base.replace(skip_layer=layers + 1)
    m = cfg.model
    w = make_weights(m, device="cuda")
    eng = Engine(cfg, w, make_tokens(cfg).cuda(), layer_kernel="fused")
    eng.step()                                   # refresh: fills every layer's K/V cache
    eng.begin_step()
    if rows < cfg.block_len:
        eng.layers_forward(0, 1)
        eng.select_active()
        l0 = 1
    else:
        l0 = 0
    n = int(eng.buffer("nrows")[0])
    assert n == rows, (n, rows)

    def fn(i):
        eng.stream = torch.cuda.current_stream()
        eng.layers_forward(l0, l0 + layers)

    t = _time(fn, reps)
    P = m.params_per_layer
    kv = 2 * m.n_kv_heads * cfg.seq_len * m.head_dim * 2
    byts = layers * (2 * P + kv)
    flops = layers * (2.0 * rows * P + 4.0 * rows * cfg.seq_len * m.n_heads * m.head_dim)
    return {"case": f"fused_m{rows}_l{layers}", "ms": t, "gbs": byts / t / 1e6, "tflops": flops / t / 1e9,
            "bytes": byts, "flops": flops}


CASES = {
    **{f"gemm_{k}_m{m}": (lambda k=k, m=m, **kw: gemm_case(k, m, **kw))
       for k in ("qkv", "o", "gu", "down") for m in (7, 32, 768)},
    "gemm_lm_m7": lambda **kw: gemm_case("lm", 7, **kw),
    "gemm_lm_m32": lambda **kw: gemm_case("lm", 32, **kw),
    "attn_m7": lambda **kw: attn_case(7, **kw),
    "attn_m32": lambda **kw: attn_case(32, **kw),
    "attn_m768": lambda **kw: attn_case(768, **kw),
    "fused_m7_l3": lambda **kw: fused_case(7, **kw),
    "fused_m32_l3": lambda **kw: fused_case(32, **kw),
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", action="append")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--bn", type=int, default=0)
    ap.add_argument("--json", action="store_true")
    a = ap.parse_args()
    names = a.case or list(CASES)
    for n in names:
        kw = {"reps": a.reps}
        if n.startswith("gemm") and "lm" not in n:
            kw.update(splits=a.splits)
            if "gu" not in n:
                kw.update(bn=a.bn)
        elif n.startswith("attn"):
            kw.update(splits=a.splits)
        r = CASES[n](**kw)
        if a.json:
            print(json.dumps(r), flush=True)
        else:
            print(f"{r['case']:>18s}  {1e3 * r['ms']:9.2f} us  {r['gbs']:8.1f} GB/s  {r['tflops']:8.1f} TFLOP/s",
                  flush=True)


if __name__ == "__main__":
    main()

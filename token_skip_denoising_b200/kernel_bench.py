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


def _copies_of(make, nbytes):
    """Enough copies of an input set that their total exceeds L2 (used round-robin)."""
    return [make(i) for i in range(_copies(nbytes))]


def score_es_case(rows, reps, d=4096):
    """ES-dLLM Eq. 1 over `rows` candidates (two fp32 hidden states per row)."""
    g = torch.Generator(device="cuda").manual_seed(3)
    nbytes = 2 * rows * d * 4
    sets = _copies_of(lambda i: (torch.randn((rows, d), generator=g, device="cuda"),
                                 torch.randn((rows, d), generator=g, device="cuda")), nbytes)
    conf = torch.rand((rows,), generator=g, device="cuda")
    mp = (torch.rand((rows,), generator=g, device="cuda") < 0.5).to(torch.uint8)
    fn = lambda i: ops.score_es(sets[i % len(sets)][0], sets[i % len(sets)][1], conf, 0.5, masked_prev=mp)
    t = _time(fn, reps)
    byts = nbytes + rows * 9
    return {"case": f"score_es_n{rows}", "ms": t, "gbs": byts / t / 1e6, "tflops": 0.0, "bytes": byts, "flops": 0}


def score_cos_case(reps, B=4, N=5120, n_resp=1024, Hkv=32, hd=128):
    """dLLM-Cache value cosine of the response rows (long-context LLaDA-8B shape, batch 4)."""
    g = torch.Generator(device="cuda").manual_seed(4)
    rows = B * n_resp
    kvd = Hkv * hd
    nbytes = rows * kvd * 4 + rows * kvd * 2
    sets = _copies_of(lambda i: (torch.randn((rows, kvd), generator=g, device="cuda"),
                                 torch.randn((B, Hkv, N, hd), generator=g, device="cuda").to(torch.bfloat16)), nbytes)
    rmap = torch.tensor([b * N + (N - n_resp) + p for b in range(B) for p in range(n_resp)], dtype=torch.int32,
                        device="cuda")
    fn = lambda i: ops.score_cos(sets[i % len(sets)][0], sets[i % len(sets)][1], rmap, N, Hkv, hd)
    t = _time(fn, reps)
    return {"case": f"score_cos_n{rows}", "ms": t, "gbs": nbytes / t / 1e6, "tflops": 0.0, "bytes": nbytes,
            "flops": 0}


def rmsnorm_case(rows, reps, d=4096):
    """Gathered RMSNorm of `rows` rows of the fp32 hidden state into the bf16 GEMM operand."""
    g = torch.Generator(device="cuda").manual_seed(5)
    nbytes = rows * d * 6
    sets = _copies_of(lambda i: torch.randn((rows, d), generator=g, device="cuda"), nbytes)
    gain = torch.ones(d, device="cuda")
    z = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
    fn = lambda i: ops.rmsnorm_rows(sets[i % len(sets)], gain, 1e-5, z=z)
    t = _time(fn, reps)
    return {"case": f"rmsnorm_m{rows}", "ms": t, "gbs": nbytes / t / 1e6, "tflops": 0.0, "bytes": nbytes,
            "flops": 0}


def select_case(n, k, reps, B=1):
    """Top-k of n scores per sequence (the ES-dLLM choice at the single-layer benchmark's size)."""
    g = torch.Generator(device="cuda").manual_seed(6)
    s = torch.rand((B * n,), generator=g, device="cuda")
    fn = lambda i: ops.select(s, B, n, ops.SEL_TOPK_DESC, k)
    t = _time(fn, reps)
    return {"case": f"select_n{n}_k{k}", "ms": t, "gbs": B * n * 4 / t / 1e6, "tflops": 0.0, "bytes": B * n * 4,
            "flops": 0}


def unmask_case(reps, B=4, N=5120, blk=64):
    """Top-1 confidence unmasking of the current block of B sequences."""
    g = torch.Generator(device="cuda").manual_seed(7)
    tokens = torch.full((B, N), 999, dtype=torch.int32, device="cuda")
    conf = torch.rand((B * N,), generator=g, device="cuda")
    amax = torch.randint(0, 998, (B * N,), generator=g, device="cuda", dtype=torch.int32)

    def fn(i):
        tokens[:, N - blk:] = 999                            # the block is masked again every call
        ops.unmask(tokens, conf, amax, N - blk, blk, 999, 1, max_out=1)
    t = _time(fn, reps)
    return {"case": f"unmask_b{B}_blk{blk}", "ms": t, "gbs": 0.0, "tflops": 0.0, "bytes": 0, "flops": 0}


def attn_gqa_case(rows, reps, N=1536, Hq=28, Hkv=4, hd=128):
    """Attention of `rows` queries over N keys, GQA 28/4 (Dream-7B shape)."""
    from synth.configs import DREAM7B
    g = torch.Generator(device="cuda").manual_seed(8)
    kvb = 2 * Hkv * N * hd * 2
    ncop = _copies(kvb)
    caches = [(torch.randn((1, Hkv, N, hd), generator=g, device="cuda").to(torch.bfloat16),
               torch.randn((1, Hkv, N, hd), generator=g, device="cuda").to(torch.bfloat16)) for _ in range(ncop)]
    q = torch.randn((rows, Hq * hd), generator=g, device="cuda").to(torch.bfloat16)
    off = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
    ws = torch.zeros(256 << 20, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    fn = lambda i: ops.attention(q, caches[i % ncop][0], caches[i % ncop][1], off, DREAM7B, rows, out=out, ws=ws)
    t = _time(fn, reps)
    byts = kvb + 2 * rows * Hq * hd * 2
    flops = 4.0 * rows * N * Hq * hd
    return {"case": f"attn_gqa_m{rows}_n{N}", "ms": t, "gbs": byts / t / 1e6, "tflops": flops / t / 1e9,
            "bytes": byts, "flops": flops}


def surelock_step_case(reps, layers=2):
    """One SureLock step of a Dream-7B-shaped model cut to `layers` layers (batch 1, prompt 256, gen
    64): the vocabulary projection of every recomputed row into stored bf16 logits, then the KL step
    (KL against the previous step's logits, confidence, locks).  Times whole steps."""
    from synth import get_config, make_tokens, make_weights
    from synth.configs import scaled
    from .engine import Engine
    cfg = scaled(get_config("dream_surelock"), n_layers=layers).replace(batch=1, prompt_len=256, gen_len=64)
    w = make_weights(cfg.model, device="cuda")
    eng = Engine(cfg, w, make_tokens(cfg).cuda())
    for _ in range(2):
        eng.step()
    torch.cuda.synchronize()
    ts = []
    for _ in range(max(3, reps // 4)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        eng.step()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    t = statistics.median(ts)
    n_lm = int(eng.buffer("nlmrows")[0])
    kl_bytes = 3 * n_lm * cfg.model.vocab * 2       # this step's logits twice, the previous step's once
    return {"case": f"surelock_step_l{layers}", "ms": t, "gbs": 0.0, "tflops": 0.0, "bytes": kl_bytes, "flops": 0,
            "lm_rows": n_lm}


def layer_case(rows, reps, N=768, dims=None):
    """One whole layer on the kernel-per-step path (the refresh path: RMSNorm, QKV + RoPE + K/V
    scatter, attention, O + residual, RMSNorm, gate/up + SwiGLU, down + residual) over `rows`
    rows of one N-position sequence, LLaDA-8B layer shape."""
    from synth import make_weights
    from synth.configs import LLADA8B, RunConfig
    from . import _lib
    m = dims or LLADA8B
    import dataclasses
    m1 = dataclasses.replace(m, n_layers=1, vocab=1024, mask_id=1023)
    run = RunConfig(name="layer", model=m1, batch=1, prompt_len=N - 64, gen_len=64, block_len=64, policy="vanilla")
    cfg = _lib.make_config(run, layer_kernel="split")
    nbytes = m1.params_per_layer * 2
    ncop = _copies(nbytes)
    ws_w = [make_weights(m1, seed=i, device="cuda", layers=[0], with_vocab=False) for i in range(ncop)]
    lws = [{k: w[k][0] for k in ("w_qkv", "w_o", "w_gu", "w_down", "g_attn", "g_ffn")} for w in ws_w]
    g = torch.Generator(device="cuda").manual_seed(9)
    h = torch.randn((N, m1.d_model), generator=g, device="cuda")
    kc = torch.randn((1, m1.n_kv_heads, N, m1.head_dim), generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn_like(kc, dtype=torch.float32).to(torch.bfloat16)
    cos, sin = ops.rope_table(N, m1.head_dim, m1.rope_theta)
    rows_t = torch.arange(rows, dtype=torch.int32, device="cuda") * (N // rows)
    cnt = torch.tensor([rows], dtype=torch.int32, device="cuda")
    off = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
    ws = torch.zeros(ops.layer_workspace_bytes(cfg, rows, rows), dtype=torch.uint8, device="cuda")
    fn = lambda i: ops.layer(cfg, lws[i % ncop], kc, vc, cos, sin, h, rows_t, cnt, off, rows, rows, ws=ws)
    t = _time(fn, reps)
    P = m1.params_per_layer
    flops = 2.0 * rows * P + 4.0 * rows * N * m1.n_heads * m1.head_dim
    byts = 2 * P + 2 * N * m1.kv_dim * 2
    return {"case": f"layer_m{rows}_n{N}", "ms": t, "gbs": byts / t / 1e6, "tflops": flops / t / 1e9,
            "bytes": byts, "flops": flops}


def gemm_epi_case(kind, rows, reps, d=4096, F=12288, splits=0, bn=0):
    """The refresh GEMMs with the epilogues the layer uses: QKV + RoPE + K/V scatter, and the
    residual add into the hidden state of O and down."""
    from synth.configs import LLADA8B
    g = torch.Generator(device="cuda").manual_seed(10)
    n_out, K = {"qkvrope": (3 * d, d), "oresid": (d, d), "downresid": (d, F)}[kind]
    nbytes = n_out * K * 2
    ncop = _copies(nbytes)
    Ws = [(torch.randn((n_out, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16) for _ in range(ncop)]
    X = torch.randn((rows, K), generator=g, device="cuda").to(torch.bfloat16)
    ws = torch.zeros(256 << 20, dtype=torch.uint8, device="cuda")
    N = rows
    rmap = torch.arange(rows, dtype=torch.int32, device="cuda")
    if kind == "qkvrope":
        cos, sin = ops.rope_table(N, 128, LLADA8B.rope_theta)
        kc = torch.zeros((1, 32, N, 128), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        fn = lambda i: ops.qkv_rope(Ws[i % ncop], X, LLADA8B, N, rmap, cos, sin, kc, vc, splits=splits, ws=ws)
        out_bytes = rows * n_out * 2
    else:
        h = torch.zeros((rows, n_out), device="cuda")
        fn = lambda i: ops.gemm(Ws[i % ncop], X, kind=3, out=h, rows_map=rmap, splits=splits, bn=bn, ws=ws)
        out_bytes = rows * n_out * 8
    t = _time(fn, reps)
    byts = nbytes + rows * K * 2 + out_bytes
    flops = 2.0 * rows * n_out * K
    return {"case": f"gemm_{kind}_m{rows}", "ms": t, "gbs": byts / t / 1e6, "tflops": flops / t / 1e9,
            "bytes": byts, "flops": flops}


CASES = {
    **{f"gemm_{k}_m{m}": (lambda k=k, m=m, **kw: gemm_case(k, m, **kw))
       for k in ("qkv", "o", "gu", "down") for m in (7, 32, 768)},
    "gemm_lm_m7": lambda **kw: gemm_case("lm", 7, **kw),
    "gemm_lm_m32": lambda **kw: gemm_case("lm", 32, **kw),
    "attn_m7": lambda **kw: attn_case(7, **kw),
    "attn_m32": lambda **kw: attn_case(32, **kw),
    "attn_m768": lambda **kw: attn_case(768, **kw),
    "attn_m5120": lambda **kw: attn_case(5120, N=5120, **kw),
    "fused_m7_l3": lambda **kw: fused_case(7, **kw),
    "fused_m32_l3": lambda **kw: fused_case(32, **kw),
    "score_es_n8192": lambda **kw: score_es_case(8192, **kw),
    "score_cos_n4096": lambda **kw: score_cos_case(**kw),
    "rmsnorm_m8192": lambda **kw: rmsnorm_case(8192, **kw),
    "select_n2048_k205": lambda **kw: select_case(2048, 205, **kw),
    "unmask_b4": lambda **kw: unmask_case(**kw),
    "attn_gqa_m1536": lambda **kw: attn_gqa_case(1536, **kw),
    "attn_gqa_m7": lambda **kw: attn_gqa_case(7, **kw),
    "surelock_step_l2": lambda **kw: surelock_step_case(**kw),
    "layer_m768": lambda **kw: layer_case(768, **kw),
    "layer_m205_n2048": lambda **kw: layer_case(205, N=2048, **kw),
    "gemm_qkvrope_m768": lambda **kw: gemm_epi_case("qkvrope", 768, **kw),
    "gemm_oresid_m768": lambda **kw: gemm_epi_case("oresid", 768, **kw),
    "gemm_downresid_m768": lambda **kw: gemm_epi_case("downresid", 768, **kw),
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
        elif n.startswith("attn") and "gqa" not in n:
            kw.update(splits=a.splits)
        r = CASES[n](**kw)
        if a.json:
            print(json.dumps(r), flush=True)
        else:
            print(f"{r['case']:>18s}  {1e3 * r['ms']:9.2f} us  {r['gbs']:8.1f} GB/s  {r['tflops']:8.1f} TFLOP/s",
                  flush=True)


if __name__ == "__main__":
    main()

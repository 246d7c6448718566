"""The persistent one-kernel layer (DLLM_LAYER_FUSED) against the kernel-per-step layer.

Both paths compute the same layer; they differ only in the order of the split-K
partial sums and so in bf16 rounding of the intermediates.  Every intermediate of
every layer of a skip step is compared, for row counts on both sides of the
16-row MMA tile, for GEMMs with fewer (tile, k-block) items than SMs and with
more, for head dims 64 and 128 and for grouped-query attention.  The oracle
comparison of whole steps runs on the default path in the step tests.
"""
import pytest
import torch

from synth import get_config, make_tokens, make_weights
from synth.configs import scaled

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from token_skip_denoising_b200.engine import Engine, device_status

TOL = 2e-2
TOL_CONF = 5e-2


def _rel(a, b):
    a, b = a.float(), b.float()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


CASES = {
    # tiny: d 256, hd 64; every GEMM has fewer items than SMs; 32 candidates, 8 kept rows
    "tiny": get_config("tiny"),
    # GQA with hd 128 (Dream-like head layout), 7 kept rows of 32
    "gqa": scaled(get_config("llada_es"), n_layers=3, d_model=1024, n_heads=8, n_kv_heads=2, head_dim=128,
                  ffn_dim=2816, vocab=2048, mask_id=2047).replace(skip_layer=1, prompt_len=96, gen_len=64),
    # LLaDA-8B layer shape, 3 layers: every GEMM has more items than SMs
    "llada": scaled(get_config("llada_es"), n_layers=3, vocab=2048, mask_id=2047).replace(skip_layer=1),
    # the widest row sets the fused kernel takes: 64 candidates, 48 kept (64-wide MMA tiles)
    "rows64": scaled(get_config("llada_es"), n_layers=2, vocab=2048, mask_id=2047).replace(
        skip_layer=1, prompt_len=64, gen_len=64, block_len=64, keep_ratio=0.75),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fused_layer_matches_split_layer(name):
    cfg = CASES[name]
    w = make_weights(cfg.model, device="cuda")
    tok0 = make_tokens(cfg).cuda()
    A = Engine(cfg, w, tok0.clone(), layer_kernel="split")
    B = Engine(cfg, w, tok0.clone(), layer_kernel="fused")
    for e in (A, B):
        e.step()                                   # refresh: all rows (split path in both)
    # From 65 rows on the refresh's O and down pieces add into h in arbitrary order, so a
    # near-tie in confidence can unmask a different token in each engine: give B exactly A's
    # state, so both layer kernels start the skip step from the same inputs.
    torch.cuda.synchronize()
    B.state.copy_(A.state)
    B.tokens.copy_(A.tokens)
    for e in (A, B):
        assert e.begin_step() == "skip"
    hd = cfg.model.head_dim
    seen = set()
    for layer in range(cfg.model.n_layers):
        if layer == cfg.skip_layer:
            A.select_active()
            B.select_active(A.buffer("scores")[:cfg.batch * cfg.block_len].clone())   # same active set
        for e in (A, B):
            e.layer_forward(layer)
        torch.cuda.synchronize()
        assert device_status() == 0
        n = int(A.buffer("nrows")[0])
        assert int(B.buffer("nrows")[0]) == n
        seen.add(n)
        rows = A.buffer("rows")[:n].long()
        assert torch.equal(B.buffer("rows")[:n].long(), rows)
        for buf in ("layer_q", "layer_attn", "layer_act"):
            assert _rel(B.buffer(buf)[:n], A.buffer(buf)[:n]) < TOL, (layer, buf)
        # the fused layer keeps the FFN operand as g * h and scales the sums by 1/rms instead:
        # the two agree up to each row's scale
        za, zb = A.buffer("layer_z")[:n].float(), B.buffer("layer_z")[:n].float()
        za = za / za.pow(2).mean(1, keepdim=True).sqrt()
        zb = zb / zb.pow(2).mean(1, keepdim=True).sqrt()
        assert _rel(zb, za) < TOL, layer
        assert _rel(B.buffer("hidden")[rows], A.buffer("hidden")[rows]) < TOL, layer
        for cache in ("kcache", "vcache"):
            assert _rel(B.buffer(cache)[layer].reshape(-1, hd), A.buffer(cache)[layer].reshape(-1, hd)) < TOL
    assert max(seen) == cfg.block_len and min(seen) == cfg.keep_count(cfg.block_len)
    for e in (A, B):
        e.unmask()
    torch.cuda.synchronize()
    # the fused sums land in a different order, so a near-tie between two confidences may
    # resolve differently: the confidences themselves are compared.  conf = exp(z_max - lse):
    # a relative error e of the hidden rows moves the logits by about e * |z| (|z| up to ~2 std
    # here), so conf carries about twice the hidden-state tolerance -- the 5e-2 that every
    # confidence comparison with the oracle uses
    assert _rel(B.buffer("conf"), A.buffer("conf")) < TOL_CONF
    assert device_status() == 0


def test_fused_layer_repeats_without_reset():
    """The phase counters clear themselves: many fused launches in a row stay correct.  Every
    candidate is kept (keep ratio 1), so a near-tie in the Eq. 1 scores cannot make the two paths
    recompute different rows."""
    cfg = CASES["tiny"].replace(keep_ratio=1.0)
    w = make_weights(cfg.model, device="cuda")
    tok0 = make_tokens(cfg).cuda()
    A = Engine(cfg, w, tok0.clone(), layer_kernel="split")
    B = Engine(cfg, w, tok0.clone(), layer_kernel="fused")
    for _ in range(5):
        A.step()
        B.step()
        torch.cuda.synchronize()
        assert device_status() == 0
        # teacher-force B onto A's decisions so the two stay on the same trajectory
        B.tokens.copy_(A.tokens)
        for buf in ("conf", "argmax", "hidden", "hprev", "masked_prev"):
            B.buffer(buf).copy_(A.buffer(buf))
        for buf in ("kcache", "vcache"):
            assert _rel(B.buffer(buf), A.buffer(buf)) < TOL
            B.buffer(buf).copy_(A.buffer(buf))


@pytest.mark.parametrize("name", ["tiny", "gqa", "llada", "rows64"])
def test_layer_runs_match_single_layers(name):
    """dllm_layers_forward (one persistent kernel per run of layers) against the split path
    layer by layer: hidden rows, every layer's K/V cache and the unmasked tokens."""
    cfg = CASES[name]
    w = make_weights(cfg.model, device="cuda")
    tok0 = make_tokens(cfg).cuda()
    A = Engine(cfg, w, tok0.clone(), layer_kernel="split")
    B = Engine(cfg, w, tok0.clone(), layer_kernel="fused")
    L, ls = cfg.model.n_layers, cfg.skip_layer
    for e in (A, B):
        e.step()
    torch.cuda.synchronize()
    B.state.copy_(A.state)                         # same inputs after an order-dependent refresh
    B.tokens.copy_(A.tokens)
    for e in (A, B):
        assert e.begin_step() == "skip"
    for layer in range(ls):
        A.layer_forward(layer)
    B.layers_forward(0, ls)
    A.select_active()
    B.select_active(A.buffer("scores")[:cfg.batch * cfg.block_len].clone())
    for layer in range(ls, L):
        A.layer_forward(layer)
    B.layers_forward(ls, L)
    torch.cuda.synchronize()
    assert device_status() == 0
    n = int(A.buffer("nrows")[0])
    rows = A.buffer("rows")[:n].long()
    assert torch.equal(B.buffer("rows")[:n].long(), rows)
    assert _rel(B.buffer("hidden")[rows], A.buffer("hidden")[rows]) < TOL
    for cache in ("kcache", "vcache"):
        for layer in range(L):
            assert _rel(B.buffer(cache)[layer], A.buffer(cache)[layer]) < TOL, (cache, layer)
    B.layers_forward(0, 0)                                    # empty run
    with pytest.raises(RuntimeError):
        B.layers_forward(1, L + 1)


def test_layer_run_in_a_cuda_graph():
    """A fused run of layers captured once and replayed gives the eager result each time."""
    cfg = CASES["llada"]
    w = make_weights(cfg.model, device="cuda")
    tok0 = make_tokens(cfg).cuda()
    E = Engine(cfg, w, tok0.clone(), layer_kernel="fused")
    E.step()
    E.begin_step()
    ls, L = cfg.skip_layer, cfg.model.n_layers
    h0 = E.buffer("hidden").clone()
    kc0, vc0 = E.buffer("kcache").clone(), E.buffer("vcache").clone()
    E.layers_forward(0, L)
    torch.cuda.synchronize()
    ref = E.buffer("hidden").clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    E.stream = s
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            E.layers_forward(0, L)
    torch.cuda.synchronize()
    for _ in range(3):
        E.buffer("hidden").copy_(h0)
        E.buffer("kcache").copy_(kc0)
        E.buffer("vcache").copy_(vc0)
        g.replay()
        torch.cuda.synchronize()
        assert device_status() == 0
        assert _rel(E.buffer("hidden"), ref) < 1e-2   # fp32 reduction order differs run to run
    E.stream = None
    del g

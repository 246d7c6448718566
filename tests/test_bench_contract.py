"""The reference arm of bench.py on the host (no GPU): one JSON line with the contract's keys,
the oracle timed on a bounded sample; under several ranks only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env):
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env.update(extra_env)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                           "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["steps"] == 2 and d["warmup"] == 3 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert "workload" in d["config"] and "model" not in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_generation_roofline_of_the_es_workload():
    """Skip steps stream every layer's weights and K/V plus the vocabulary projection (HBM-bound);
    refreshes recompute all 768 rows (tensor-bound at these peaks)."""
    sys.path.insert(0, ROOT)
    import bench
    from synth import get_config
    cfg = get_config("llada_es")
    m = cfg.model
    peaks = {"hbm_gbs": 6650.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    r = bench.generation_roofline(cfg, peaks, 1000.0)
    P = m.params_per_layer
    weights = m.n_layers * 2 * P + 2 * m.vocab * m.d_model
    kv = m.n_layers * 2 * cfg.batch * cfg.seq_len * m.kv_dim * 2
    assert abs(r["skip_step"]["bytes"] / (weights + kv) - 1) < 2e-3      # row traffic is the small rest
    assert r["skip_step"]["bound"] == "hbm" and r["refresh_step"]["bound"] == "tensor"
    refresh_flops = 2 * cfg.seq_len * P * m.n_layers + 4 * cfg.seq_len * cfg.seq_len * m.n_heads * m.head_dim * m.n_layers
    assert abs(r["refresh_step"]["flops"] / (refresh_flops + 2 * cfg.block_len * m.vocab * m.d_model) - 1) < 1e-9
    assert r["skip_step"]["count"] == 248 and r["refresh_step"]["count"] == 8
    want_ms = 248 * r["skip_step"]["bytes"] / 6650e6 + 8 * r["refresh_step"]["flops"] / 1400e9
    assert abs(r["roofline_ms"] - want_ms) < 0.01 and abs(r["frac"] - r["roofline_ms"] / 1000.0) < 1e-4
    assert bench.whole_job_tokens_per_s(1, 256, 3, 2, 2.0) == 1 * 256 * 3 * 2 / 2.0

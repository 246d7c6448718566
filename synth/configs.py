"""The five workloads: model shapes, generation schedule and selection policy.

Values are the stated configurations of the token-skipping denoising step
(a tiny fp32 model, a single-layer microbenchmark, an LLaDA-8B shape with
ES-dLLM, a Dream-7B shape with SureLock, and a long-context LLaDA-8B shape with
dLLM-Cache + DUS).  Where a configuration is silent the value below is the
plain reading (RoPE theta 10000, RMSNorm eps 1e-5, mask id V-1, alpha 0.5).
"""
from __future__ import annotations

import dataclasses
import math

POLICY_VANILLA = "vanilla"
POLICY_ES = "es"
POLICY_SURELOCK = "surelock"
POLICY_DLLM_CACHE = "dllm_cache"

UNMASK_TOPCONF = "topconf"
UNMASK_DUS = "dus"
UNMASK_CB_DUS = "cb_dus"   # confidence-bounded, filtered by the dilation (non-adjacency) rule

SCOPE_BLOCK = "block"   # candidates = rows of the current block
SCOPE_ALL = "all"       # candidates = every row of the sequence


@dataclasses.dataclass(frozen=True)
class ModelDims:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    vocab: int
    mask_id: int
    rope_theta: float = 10000.0
    rms_eps: float = 1e-5

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def qkv_dim(self) -> int:
        return self.q_dim + 2 * self.kv_dim

    @property
    def params_per_layer(self) -> int:
        d = self.d_model
        return d * self.qkv_dim + self.q_dim * d + 3 * d * self.ffn_dim


@dataclasses.dataclass(frozen=True)
class RunConfig:
    name: str
    model: ModelDims
    batch: int
    prompt_len: int
    gen_len: int
    block_len: int
    policy: str = POLICY_ES
    unmask: str = UNMASK_TOPCONF
    tokens_per_step: int = 1
    # ES-dLLM
    skip_layer: int = 1
    keep_ratio: float = 1.0
    alpha: float = 0.5
    cand_scope: str = SCOPE_BLOCK
    refresh_period: int = 0          # 0: refresh only at the first step of a block
    es_per_layer: bool = False       # re-select the top k at every layer from skip_layer on
    # SureLock
    kl_eps: float = 1e-3
    conf_tau: float = 0.9
    lock_masked: bool = False        # SureLock: masked positions may lock too
    # dLLM-Cache
    sim_tau: float = 0.95
    rho_cap: float = 0.25
    prompt_interval: int = 50
    # DUS
    dus_base: int = 2
    # confidence-bounded unmasking (unmask = cb_dus): take tokens with confidence >= cb_tau,
    # at most tokens_per_step, none next to another taken in the same step
    cb_tau: float = 0.9

    @property
    def seq_len(self) -> int:
        return self.prompt_len + self.gen_len

    @property
    def n_blocks(self) -> int:
        return self.gen_len // self.block_len

    def replace(self, **kw) -> "RunConfig":
        return dataclasses.replace(self, **kw)

    def keep_count(self, n: int) -> int:
        """k = ceil(keep_ratio * n) clamped to [1, n] (the pages leave rounding open)."""
        if n <= 0:
            return 0
        return max(1, min(n, math.ceil(self.keep_ratio * n - 1e-9)))


TINY = ModelDims(n_layers=2, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64,
                 ffn_dim=1024, vocab=1024, mask_id=1023, rope_theta=10000.0)

MICRO = ModelDims(n_layers=1, d_model=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                  ffn_dim=12288, vocab=1024, mask_id=1023, rope_theta=10000.0)

LLADA8B = ModelDims(n_layers=32, d_model=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                    ffn_dim=12288, vocab=126464, mask_id=126463, rope_theta=500000.0)

DREAM7B = ModelDims(n_layers=28, d_model=3584, n_heads=28, n_kv_heads=4, head_dim=128,
                    ffn_dim=18944, vocab=152064, mask_id=152063, rope_theta=10000.0)

MICRO_RHOS = (0.03, 0.1, 0.25, 0.5, 1.0)

CONFIGS = {
    # 1: tiny model, the whole generation runs on the oracle in seconds
    "tiny": RunConfig(name="tiny", model=TINY, batch=1, prompt_len=32, gen_len=32,
                      block_len=32, policy=POLICY_ES, tokens_per_step=4,
                      skip_layer=1, keep_ratio=0.25, alpha=0.5),
    # 2: single-layer microbenchmark, N = 2048 rows; prompt_len 0 (all rows are candidates)
    "micro": RunConfig(name="micro", model=MICRO, batch=1, prompt_len=0, gen_len=2048,
                       block_len=2048, policy=POLICY_ES, skip_layer=0, keep_ratio=0.25,
                       alpha=0.5, cand_scope=SCOPE_ALL),
    # 3: LLaDA-8B shape, ES-dLLM skip at layer 4 keeping 20% of the block
    "llada_es": RunConfig(name="llada_es", model=LLADA8B, batch=1, prompt_len=512,
                          gen_len=256, block_len=32, policy=POLICY_ES, tokens_per_step=1,
                          skip_layer=4, keep_ratio=0.2, alpha=0.5),
    # 4: Dream-7B shape, SureLock
    "dream_surelock": RunConfig(name="dream_surelock", model=DREAM7B, batch=8,
                                prompt_len=1024, gen_len=512, block_len=32,
                                policy=POLICY_SURELOCK, tokens_per_step=1,
                                kl_eps=1e-3, conf_tau=0.9),
    # 5: long-context LLaDA-8B shape, dLLM-Cache + DUS
    "llada_cache_dus": RunConfig(name="llada_cache_dus", model=LLADA8B, batch=4,
                                 prompt_len=4096, gen_len=1024, block_len=64,
                                 policy=POLICY_DLLM_CACHE, unmask=UNMASK_DUS,
                                 sim_tau=0.95, rho_cap=0.25, prompt_interval=50),
}


def get_config(name: str) -> RunConfig:
    return CONFIGS[name]


def scaled(cfg: RunConfig, **model_kw) -> RunConfig:
    """The same run with a smaller model (parity cases that the oracle finishes quickly)."""
    return cfg.replace(model=dataclasses.replace(cfg.model, **model_kw))

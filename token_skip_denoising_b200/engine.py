"""Python face of the C ABI: the generation engine and single-kernel ops.

Only argument marshalling happens here.  torch provides device memory and the
stream; every step of the denoising path runs in libdllm.so.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import check, ptr, stream_ptr


def _weights_struct(w: dict) -> _lib.DllmWeights:
    s = _lib.DllmWeights()
    for k in ("embed", "lm_head", "w_qkv", "w_o", "w_gu", "w_down", "g_attn", "g_ffn", "g_final"):
        t = w[k]
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"weight {k} must be a contiguous CUDA tensor")
        setattr(s, k, t.data_ptr())
    return s


def state_bytes(cfg: _lib.DllmConfig):
    lib = _lib.load()
    sb, wb = ctypes.c_size_t(), ctypes.c_size_t()
    check(lib.dllm_state_bytes(ctypes.byref(cfg), ctypes.byref(sb), ctypes.byref(wb)), "dllm_state_bytes")
    return sb.value, wb.value


class Engine:
    """One generation over a batch: owns the state/workspace tensors and the handle.

    run: a synth.RunConfig; weights: dict of CUDA tensors in the library layout;
    tokens: CUDA int32 [B, N] (prompt then mask ids), updated in place.
    """

    def __init__(self, run, weights: dict, tokens: torch.Tensor, stream=None, **cfg_over):
        self.lib = _lib.load()
        self.run = run
        self.cfg = _lib.make_config(run, **cfg_over)
        self.weights = weights
        if tokens.dtype != torch.int32 or not tokens.is_cuda:
            raise ValueError("tokens must be a CUDA int32 tensor")
        self.tokens = tokens
        self.stream = stream
        sb, wb = state_bytes(self.cfg)
        self.state = torch.empty(sb, dtype=torch.uint8, device="cuda")
        self.workspace = torch.empty(wb, dtype=torch.uint8, device="cuda")
        self._w = _weights_struct(weights)
        h = ctypes.c_void_p()
        check(self.lib.dllm_step_init(ctypes.byref(h), ctypes.byref(self.cfg), ctypes.byref(self._w),
                                      self.state.data_ptr(), self.workspace.data_ptr(), tokens.data_ptr(),
                                      stream_ptr(stream)), "dllm_step_init")
        self.handle = h

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self.lib.dllm_destroy(h)
            self.handle = None

    @property
    def done(self) -> bool:
        return bool(self.lib.dllm_done(self.handle))

    def step(self, info: bool = False):
        si = _lib.DllmStepInfo() if info else None
        check(self.lib.dllm_step(self.handle, ctypes.byref(si) if info else None, stream_ptr(self.stream)),
              "dllm_step")
        if info:
            return {f: getattr(si, f) for f, _ in si._fields_} | {"kind_name": _lib.STEP_KIND[si.kind]}
        return None

    def begin_step(self) -> str:
        k = ctypes.c_int32()
        check(self.lib.dllm_begin_step(self.handle, ctypes.byref(k), stream_ptr(self.stream)), "dllm_begin_step")
        return _lib.STEP_KIND[k.value]

    def layer_forward(self, layer: int):
        check(self.lib.dllm_layer_forward(self.handle, layer, stream_ptr(self.stream)), "dllm_layer_forward")

    def layers_forward(self, l0: int, l1: int):
        """Layers l0 .. l1-1 for the current row set (one persistent kernel when it applies)."""
        check(self.lib.dllm_layers_forward(self.handle, l0, l1, stream_ptr(self.stream)), "dllm_layers_forward")

    def select_active(self, scores: torch.Tensor | None = None, active_idx=None, active_count=None):
        check(self.lib.dllm_select_active(self.handle, ptr(scores), ptr(active_idx), ptr(active_count),
                                          stream_ptr(self.stream)), "dllm_select_active")

    def select_layers_forward(self, scores: torch.Tensor | None = None):
        """Per-layer ES: every layer from the skip layer on, each after its own choice
        (scores: optional fp32 [L - skip_layer, B, n_cand] used for the choices)."""
        check(self.lib.dllm_select_layers_forward(self.handle, ptr(scores), stream_ptr(self.stream)),
              "dllm_select_layers_forward")

    def unmask(self, pos_out=None, tok_out=None, n_out=None):
        check(self.lib.dllm_unmask(self.handle, ptr(pos_out), ptr(tok_out), ptr(n_out), stream_ptr(self.stream)),
              "dllm_unmask")

    def reset(self, tokens: torch.Tensor | None = None):
        """Rewind to a new generation (tokens, if given, are copied in first)."""
        if tokens is not None:
            self.tokens.copy_(tokens, non_blocking=True)
        check(self.lib.dllm_reset(self.handle, stream_ptr(self.stream)), "dllm_reset")

    def set_lock_pattern(self, pattern: torch.Tensor | None):
        """SureLock measurement mode: lock rows by a seeded pattern (uint8 [B, N] on the device)."""
        self._lock_pattern = pattern
        check(self.lib.dllm_set_lock_pattern(self.handle, ptr(pattern)), "dllm_set_lock_pattern")

    def set_forced_similarities(self, sims: torch.Tensor | None):
        """dLLM-Cache teacher forcing: per-layer similarities fp32 [L, B, n_resp] on the device."""
        self._forced_sims = sims
        check(self.lib.dllm_set_forced_similarities(self.handle, ptr(sims)), "dllm_set_forced_similarities")

    def set_wait_limit(self, polls: int):
        """Poll limit of the fused layer kernel's grid-phase waits (0: the default)."""
        check(self.lib.dllm_set_wait_limit(self.handle, int(polls)), "dllm_set_wait_limit")

    def progress(self) -> dict:
        """Schedule position (with the state buffer and the tokens: the whole generation state)."""
        p = _lib.DllmProgress()
        check(self.lib.dllm_get_progress(self.handle, ctypes.byref(p)), "dllm_get_progress")
        return {f: getattr(p, f) for f, _ in p._fields_}

    def set_progress(self, prog: dict):
        p = _lib.DllmProgress(**prog)
        check(self.lib.dllm_set_progress(self.handle, ctypes.byref(p)), "dllm_set_progress")

    def profile(self, every: int, hbm_gbs: float = 0.0, tensor_tflops: float = 0.0):
        """Bracket every `every`-th GEMM / attention launch with CUDA events (0: off)."""
        check(self.lib.dllm_profile_enable(self.handle, int(every), hbm_gbs, tensor_tflops),
              "dllm_profile_enable")

    def profile_read(self) -> dict:
        p = _lib.DllmProfile()
        check(self.lib.dllm_profile_read(self.handle, ctypes.byref(p)), "dllm_profile_read")
        return {f: getattr(p, f) for f, _ in p._fields_}

    def generate(self):
        while not self.done:
            self.step()

    def buffer(self, name: str, dtype=None, shape=None) -> torch.Tensor:
        """A view of an internal device buffer (see DLLM_BUF_* in include/dllm.h)."""
        p, nb = ctypes.c_void_p(), ctypes.c_size_t()
        check(self.lib.dllm_get_buffer(self.handle, _lib.BUF[name], ctypes.byref(p), ctypes.byref(nb)),
              "dllm_get_buffer")
        if not p.value:
            raise ValueError(f"buffer {name} is not allocated for this policy")
        c = self.cfg
        B, N = c.batch, c.prompt_len + c.gen_len
        defaults = {
            "kcache": (torch.bfloat16, (c.n_layers, B, c.n_kv_heads, N, c.head_dim)),
            "vcache": (torch.bfloat16, (c.n_layers, B, c.n_kv_heads, N, c.head_dim)),
            "hidden": (torch.float32, (B * N, c.d_model)), "hprev": (torch.float32, (B * N, c.d_model)),
            "conf": (torch.float32, (B * N,)), "argmax": (torch.int32, (B * N,)),
            "rows": (torch.int32, (B * N,)), "nrows": (torch.int32, (1,)),
            "scores": (torch.float32, (B * N,)), "lock": (torch.uint8, (B * N,)),
            "masked_prev": (torch.uint8, (B * N,)), "lmrows": (torch.int32, (B * N,)),
            "nlmrows": (torch.int32, (1,)), "kl": (torch.float32, (B * N,)),
            "hcache": (torch.float32, (c.n_layers, B * N, c.d_model)), "lse": (torch.float32, (B * N,)),
            "selrows": (torch.int32, (B * N,)), "nsel": (torch.int32, (1,)),
            "layer_z": (torch.bfloat16, (-1, c.d_model)), "layer_q": (torch.bfloat16, (-1, c.n_heads * c.head_dim)),
            "layer_attn": (torch.bfloat16, (-1, c.n_heads * c.head_dim)),
            "layer_act": (torch.bfloat16, (-1, c.ffn_dim)),
            "es_in": (torch.float32, (-1, B * N, c.d_model)),
            "zstore": (torch.bfloat16, (2, B * N, c.vocab)), "lse_store": (torch.float32, (2, B * N)),
            "stamp": (torch.int32, (B * N,)),
            "vnew": (torch.float32, (-1, c.n_kv_heads * c.head_dim)),
            "fused_sync": (torch.int32, (16,)),
        }
        dt, shp = defaults[name]
        if shape is None and shp[0] == -1:
            inner = 1
            for v in shp[1:]:
                inner *= v
            shp = (nb.value // (inner * torch.empty(0, dtype=dt).element_size()),) + tuple(shp[1:])
        return _lib.view(p.value, shape or shp, dtype or dt)


def device_status(reset: bool = True) -> int:
    lib = _lib.load()
    v = ctypes.c_int32()
    check(lib.dllm_device_status(ctypes.byref(v), 1 if reset else 0), "dllm_device_status")
    return v.value


def kernel_launches() -> int:
    return int(_lib.load().dllm_kernel_launches())

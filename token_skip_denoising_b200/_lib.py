"""ctypes binding of libdllm.so: argument marshalling only.

Every computation runs in the CUDA library; this module converts torch
tensors (device memory owned by the caller) to pointers and checks status
codes.  A missing or unloadable library raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdllm.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "dllm.h")

c_i32 = ctypes.c_int32
c_f32 = ctypes.c_float
c_f64 = ctypes.c_double
c_vp = ctypes.c_void_p
c_sz = ctypes.c_size_t
P = ctypes.POINTER

DLLM_OK = 0
STATUS_NAMES = {0: "DLLM_OK", 1: "DLLM_ERR_INVALID_ARG", 2: "DLLM_ERR_SHAPE", 3: "DLLM_ERR_UNSUPPORTED",
                4: "DLLM_ERR_CUDA", 5: "DLLM_ERR_TIMEOUT", 6: "DLLM_ERR_DEVICE", 7: "DLLM_ERR_STATE"}
POLICY = {"vanilla": 0, "es": 1, "surelock": 2, "dllm_cache": 3}
UNMASK = {"topconf": 0, "dus": 1, "cb_dus": 2}
SCOPE = {"block": 0, "all": 1}
STEP_KIND = {0: "full", 1: "skip", 2: "locked", 3: "partial"}
BUF = {"kcache": 0, "vcache": 1, "hidden": 2, "hprev": 3, "conf": 4, "argmax": 5, "rows": 6, "nrows": 7,
       "scores": 8, "lock": 9, "masked_prev": 10, "lmrows": 11, "nlmrows": 12, "kl": 13, "hcache": 14, "lse": 15,
       "selrows": 16, "nsel": 17, "layer_z": 18, "layer_q": 19, "layer_attn": 20, "layer_act": 21,
       "es_in": 22, "zstore": 23, "lse_store": 24, "stamp": 25, "vnew": 26, "fused_sync": 27}
LAYER_KERNEL = {"auto": 0, "split": 1, "fused": 2}


class DllmConfig(ctypes.Structure):
    _fields_ = [("n_layers", c_i32), ("d_model", c_i32), ("n_heads", c_i32), ("n_kv_heads", c_i32),
                ("head_dim", c_i32), ("ffn_dim", c_i32), ("vocab", c_i32), ("mask_id", c_i32),
                ("rope_theta", c_f32), ("rms_eps", c_f32),
                ("batch", c_i32), ("prompt_len", c_i32), ("gen_len", c_i32), ("block_len", c_i32),
                ("policy", c_i32), ("cand_scope", c_i32),
                ("skip_layer", c_i32), ("keep_ratio", c_f32), ("alpha", c_f32), ("refresh_period", c_i32),
                ("kl_eps", c_f32), ("conf_tau", c_f32),
                ("sim_tau", c_f32), ("rho_cap", c_f32), ("prompt_interval", c_i32), ("forced_rho", c_i32),
                ("unmask", c_i32), ("tokens_per_step", c_i32), ("layer_kernel", c_i32), ("lock_masked", c_i32),
                ("cb_tau", c_f32), ("es_per_layer", c_i32)]


class DllmWeights(ctypes.Structure):
    _fields_ = [("embed", c_vp), ("lm_head", c_vp), ("w_qkv", c_vp), ("w_o", c_vp), ("w_gu", c_vp),
                ("w_down", c_vp), ("g_attn", c_vp), ("g_ffn", c_vp), ("g_final", c_vp)]


class DllmStepInfo(ctypes.Structure):
    _fields_ = [("kind", c_i32), ("step", c_i32), ("block", c_i32), ("step_in_block", c_i32),
                ("rows_first", c_i32), ("rows_last", c_i32), ("lm_rows", c_i32), ("n_locked", c_i32),
                ("done", c_i32)]


class DllmProgress(ctypes.Structure):
    _fields_ = [("step", c_i32), ("block", c_i32), ("step_in_block", c_i32)]


class DllmProfile(ctypes.Structure):
    _fields_ = [("gemm_launches", ctypes.c_int64), ("gemm_ms", c_f64), ("gemm_bytes", c_f64), ("gemm_flops", c_f64),
                ("gemm_roofline_ms", c_f64), ("attn_launches", ctypes.c_int64), ("attn_ms", c_f64),
                ("attn_bytes", c_f64), ("attn_flops", c_f64), ("fused_launches", ctypes.c_int64),
                ("fused_layers", ctypes.c_int64), ("fused_ms", c_f64), ("fused_bytes", c_f64), ("fused_flops", c_f64)]


_SIGS = {
    "dllm_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "dllm_last_error": (ctypes.c_char_p, []),
    "dllm_device_status": (ctypes.c_int, [P(c_i32), c_i32]),
    "dllm_state_bytes": (ctypes.c_int, [P(DllmConfig), P(c_sz), P(c_sz)]),
    "dllm_step_init": (ctypes.c_int, [P(c_vp), P(DllmConfig), P(DllmWeights), c_vp, c_vp, c_vp, c_vp]),
    "dllm_begin_step": (ctypes.c_int, [c_vp, P(c_i32), c_vp]),
    "dllm_layer_forward": (ctypes.c_int, [c_vp, c_i32, c_vp]),
    "dllm_layers_forward": (ctypes.c_int, [c_vp, c_i32, c_i32, c_vp]),
    "dllm_select_active": (ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp]),
    "dllm_select_layers_forward": (ctypes.c_int, [c_vp, c_vp, c_vp]),
    "dllm_unmask": (ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp]),
    "dllm_step": (ctypes.c_int, [c_vp, P(DllmStepInfo), c_vp]),
    "dllm_done": (ctypes.c_int, [c_vp]),
    "dllm_reset": (ctypes.c_int, [c_vp, c_vp]),
    "dllm_set_lock_pattern": (ctypes.c_int, [c_vp, c_vp]),
    "dllm_profile_enable": (ctypes.c_int, [c_vp, c_i32, c_f64, c_f64]),
    "dllm_profile_read": (ctypes.c_int, [c_vp, P(DllmProfile)]),
    "dllm_get_progress": (ctypes.c_int, [c_vp, P(DllmProgress)]),
    "dllm_set_progress": (ctypes.c_int, [c_vp, P(DllmProgress)]),
    "dllm_set_forced_similarities": (ctypes.c_int, [c_vp, c_vp]),
    "dllm_set_wait_limit": (ctypes.c_int, [c_vp, ctypes.c_uint32]),
    "dllm_kernel_launches": (ctypes.c_int64, []),
    "dllm_get_buffer": (ctypes.c_int, [c_vp, c_i32, P(c_vp), P(c_sz)]),
    "dllm_destroy": (None, [c_vp]),
    "dllm_op_rope_table": (ctypes.c_int, [c_vp, c_vp, c_i32, c_i32, c_f64, c_vp]),
    "dllm_op_embed_rows": (ctypes.c_int, [c_vp, c_i32, c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_vp]),
    "dllm_op_rmsnorm_rows": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_f32, c_vp, c_vp]),
    "dllm_op_gemm": (ctypes.c_int, [c_i32, c_vp, c_i32, c_vp, c_i32, c_vp, c_i32, c_vp, c_vp, c_i32, c_i32,
                                    c_vp, c_sz, c_vp]),
    "dllm_op_gemm_noalloc": (ctypes.c_int, [c_i32, c_vp, c_i32, c_vp, c_i32, c_vp, c_i32, c_vp, c_vp, c_vp]),
    "dllm_op_qkv_rope": (ctypes.c_int, [c_vp, c_vp, c_i32, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp,
                                        c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_sz, c_vp]),
    "dllm_op_gate_up": (ctypes.c_int, [c_vp, c_i32, c_vp, c_i32, c_vp, c_i32, c_vp, c_i32, c_vp, c_sz, c_vp]),
    "dllm_op_attention": (ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                         c_i32, c_i32, c_vp, c_sz, c_vp]),
    "dllm_op_lm_head": (ctypes.c_int, [c_vp, c_i32, c_vp, c_i32, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp,
                                       c_vp, c_sz, c_vp]),
    "dllm_op_score_es": (ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_i32, c_i32, c_f32, c_i32,
                                        c_vp, c_vp]),
    "dllm_op_score_cos": (ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp]),
    "dllm_op_kl_conf": (ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_vp, c_vp,
                                       c_vp, c_vp, c_vp]),
    "dllm_op_select": (ctypes.c_int, [c_vp, c_i32, c_i32, c_i32, c_i32, c_f32, c_i32, c_i32, c_vp, c_vp, c_i32,
                                      c_vp, c_vp, c_vp, c_vp]),
    "dllm_op_unmask": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_f32,
                                      c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp]),
    "dllm_op_layer": (ctypes.c_int, [P(DllmConfig), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                     c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_sz, c_vp]),
    "dllm_op_layer_workspace": (ctypes.c_int, [P(DllmConfig), c_i32, c_i32, P(c_sz)]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libdllm.so and declare every prototype; raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libdllm.so not built at {path}: run token_skip_denoising_b200/build.py")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def header_symbols(path: str = HEADER):
    """Function names declared in include/dllm.h."""
    text = open(path).read()
    return sorted(set(re.findall(r"\b(dllm_\w+)\s*\(", text)) - {"dllm_handle"})


class DllmError(RuntimeError):
    def __init__(self, rc, where):
        lib = load()
        msg = lib.dllm_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(rc, rc)} ({lib.dllm_status_string(rc).decode()}): {msg}")
        self.status = rc


def check(rc: int, where: str = "dllm"):
    if rc != DLLM_OK:
        raise DllmError(rc, where)


def ptr(t) -> int:
    """Device address of a tensor (None -> NULL)."""
    return None if t is None else t.data_ptr()


def stream_ptr(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_config(run, **over) -> DllmConfig:
    """A DllmConfig from a synth.RunConfig (field names match)."""
    m = run.model
    c = DllmConfig()
    c.n_layers, c.d_model, c.n_heads, c.n_kv_heads = m.n_layers, m.d_model, m.n_heads, m.n_kv_heads
    c.head_dim, c.ffn_dim, c.vocab, c.mask_id = m.head_dim, m.ffn_dim, m.vocab, m.mask_id
    c.rope_theta, c.rms_eps = m.rope_theta, m.rms_eps
    c.batch, c.prompt_len, c.gen_len, c.block_len = run.batch, run.prompt_len, run.gen_len, run.block_len
    c.policy = POLICY[run.policy]
    c.cand_scope = SCOPE[run.cand_scope]
    c.skip_layer, c.keep_ratio, c.alpha = run.skip_layer, run.keep_ratio, run.alpha
    c.refresh_period = run.refresh_period
    c.kl_eps, c.conf_tau = run.kl_eps, run.conf_tau
    c.sim_tau, c.rho_cap, c.prompt_interval = run.sim_tau, run.rho_cap, run.prompt_interval
    c.forced_rho = 0
    c.unmask = UNMASK[run.unmask]
    c.tokens_per_step = run.tokens_per_step
    c.layer_kernel = 0
    c.lock_masked = 1 if run.lock_masked else 0
    c.cb_tau = run.cb_tau
    c.es_per_layer = 1 if run.es_per_layer else 0
    for k, v in over.items():
        if k == "layer_kernel" and isinstance(v, str):
            v = LAYER_KERNEL[v]
        setattr(c, k, v)
    return c


class _CudaArray:
    def __init__(self, p, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (p, False),
                                         "version": 3, "strides": None}


def view(p: int, shape, dtype):
    """A torch tensor aliasing device memory at address p (no copy)."""
    import torch
    typestr = {torch.float32: "<f4", torch.int32: "<i4", torch.uint8: "|u1", torch.bfloat16: "<f2",
               torch.float16: "<f2"}[dtype]
    if dtype == torch.bfloat16:
        t = torch.as_tensor(_CudaArray(p, shape, "<i2"), device="cuda")
        return t.view(torch.bfloat16)
    return torch.as_tensor(_CudaArray(p, shape, typestr), device="cuda")

"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and validates configurations on the host (no GPU needed)."""
import ctypes

import pytest

from synth import get_config
from token_skip_denoising_b200 import _lib


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_exports_every_declared_symbol(lib):
    declared = _lib.header_symbols()
    assert len(declared) >= 25
    missing = [s for s in declared if not hasattr(lib, s)]
    assert not missing, missing
    # and the binding declares a prototype for each of them
    assert set(declared) <= set(_lib._SIGS)


def test_status_strings(lib):
    assert lib.dllm_status_string(0) == b"ok"
    assert lib.dllm_status_string(3) == b"unsupported"
    assert lib.dllm_status_string(99) == b"unknown status"


@pytest.mark.parametrize("name", ["tiny", "micro", "llada_es", "dream_surelock", "llada_cache_dus"])
def test_state_bytes_for_every_workload(lib, name):
    cfg = _lib.make_config(get_config(name))
    sb, wb = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.dllm_state_bytes(ctypes.byref(cfg), ctypes.byref(sb), ctypes.byref(wb)) == 0, \
        lib.dllm_last_error()
    assert sb.value > 0 and wb.value > 0
    assert sb.value < 120e9 and wb.value < 20e9      # fits beside the weights in 180 GB


def test_state_bytes_covers_kv_cache(lib):
    run = get_config("llada_es")
    m = run.model
    cfg = _lib.make_config(run)
    sb, wb = ctypes.c_size_t(), ctypes.c_size_t()
    lib.dllm_state_bytes(ctypes.byref(cfg), ctypes.byref(sb), ctypes.byref(wb))
    kv = 2 * m.n_layers * run.batch * m.n_kv_heads * run.seq_len * m.head_dim * 2
    assert sb.value >= kv


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, 3), ("gen_len", 33, 2), ("n_kv_heads", 3, 2), ("mask_id", 5000, 1),
    ("policy", 9, 1), ("keep_ratio", 0.0, 1), ("skip_layer", 99, 1), ("vocab", 1000, 3),
    ("es_per_layer", 2, 1), ("lock_masked", 2, 1), ("layer_kernel", 7, 1), ("unmask", 9, 1),
])
def test_invalid_configs_are_rejected(lib, field, value, status):
    cfg = _lib.make_config(get_config("tiny"))
    setattr(cfg, field, value)
    if field == "vocab":
        cfg.mask_id = value - 1
    sb, wb = ctypes.c_size_t(), ctypes.c_size_t()
    rc = lib.dllm_state_bytes(ctypes.byref(cfg), ctypes.byref(sb), ctypes.byref(wb))
    assert rc == status, (rc, lib.dllm_last_error())
    assert lib.dllm_last_error()


def test_dus_block_of_two_rejected(lib):
    run = get_config("tiny").replace(unmask="dus", block_len=2)
    cfg = _lib.make_config(run)
    sb, wb = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.dllm_state_bytes(ctypes.byref(cfg), ctypes.byref(sb), ctypes.byref(wb)) == 3


def test_null_arguments_are_rejected_without_a_gpu(lib):
    assert lib.dllm_state_bytes(None, None, None) == 1
    h = ctypes.c_void_p()
    cfg = _lib.make_config(get_config("tiny"))
    assert lib.dllm_step_init(ctypes.byref(h), ctypes.byref(cfg), None, None, None, None, None) == 1
    assert lib.dllm_op_select(None, 1, 4, 0, 2, 0.0, 0, 4, None, None, 0, None, None, None, None) == 1


def test_qkv_rope_rejects_misaligned_tables_and_caches_before_any_launch(lib):
    # the RoPE pass moves 16-byte table rows and 8-byte groups of q / cache elements; the op
    # checks the caller's pointers on the host first (these addresses are never dereferenced)
    base = 1 << 20
    args = lambda cos, kc: (base, base, 16, None, 256, 4, 4, 64, 32, base, cos, base, base, kc, base, 0,
                            base, 1 << 24, None)
    assert lib.dllm_op_qkv_rope(*args(base + 8, base)) == 1       # cos table on an 8-byte boundary
    assert lib.dllm_op_qkv_rope(*args(base, base + 2)) == 1       # K cache on a 2-byte boundary
    ok = args(base, base)
    assert lib.dllm_op_qkv_rope(*ok[:5], 1, *ok[6:]) == 2          # one 64-wide q head: not a multiple of 128


def test_misaligned_operands_are_refused_before_any_launch(lib):
    # every kernel moves 16-byte (some 8-byte) vectors; each entry point checks the caller's
    # pointers on the host first, so these addresses are never dereferenced
    A = 1 << 20                                   # a 256-byte aligned stand-in address
    assert lib.dllm_op_embed_rows(A, 1024, A, A, None, 4, 256, A + 4, None) == 1
    assert lib.dllm_op_embed_rows(A + 8, 1024, A, A, None, 4, 256, A, None) == 1
    assert lib.dllm_op_rmsnorm_rows(A, A, None, 4, 256, A, 1e-5, A + 2, None) == 1
    assert lib.dllm_op_rmsnorm_rows(A, A, None, 4, 256, A + 4, 1e-5, A, None) == 1
    assert lib.dllm_op_score_es(A, A + 4, A, None, None, 0, None, 4, 256, 0.5, 0, A, None) == 1
    assert lib.dllm_op_attention(A + 8, A, A, A, A, 1, 4, 4, 64, 4, 4, 128, 1, A, 1 << 20, None) == 1
    assert lib.dllm_op_attention(A, A, A + 2, A, A, 1, 4, 4, 64, 4, 4, 128, 1, A, 1 << 20, None) == 1
    assert lib.dllm_op_gemm(0, A, 128, A, 4, None, 256, A, None, 0, 0, A + 16, 1 << 24, None) == 1
    cfg = _lib.make_config(get_config("tiny"))
    op = lambda kc, ws: lib.dllm_op_layer(ctypes.byref(cfg), A, A, A, A, A, A, kc, A, A, A, A, A, A, A, 4, 4,
                                          ws, 1 << 30, None)
    assert op(A + 8, A) == 1                      # K cache on an 8-byte boundary
    assert op(A, A + 16) == 1                     # workspace not 256-byte aligned
    w = _lib.DllmWeights(A, A, A, A + 2, A, A, A, A, A)
    h = ctypes.c_void_p()
    assert lib.dllm_step_init(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(w), A, A, A, None) == 1
    w = _lib.DllmWeights(A, A, A, A, A, A, A, A, A)
    assert lib.dllm_step_init(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(w), A, A, A + 2, None) == 1
    assert not h.value                            # no handle was made


def test_per_layer_selection_needs_a_layer_after_the_skip_layer(lib):
    run = get_config("tiny").replace(es_per_layer=True)
    sb, wb = ctypes.c_size_t(), ctypes.c_size_t()
    cfg = _lib.make_config(run.replace(skip_layer=run.model.n_layers))
    assert lib.dllm_state_bytes(ctypes.byref(cfg), ctypes.byref(sb), ctypes.byref(wb)) == 1
    cfg = _lib.make_config(run.replace(skip_layer=run.model.n_layers - 1))
    assert lib.dllm_state_bytes(ctypes.byref(cfg), ctypes.byref(sb), ctypes.byref(wb)) == 0


def test_per_layer_state_holds_one_input_snapshot_per_layer_above_the_skip_layer(lib):
    # the per-layer choice keeps, for every layer above the skip layer, each row's input of
    # that layer last iteration: (L - L_s - 1) fp32 [B*N, d] slabs more than the per-step choice
    run = get_config("llada_es")
    m = run.model
    sizes = []
    for per_layer in (False, True):
        cfg = _lib.make_config(run.replace(es_per_layer=per_layer))
        sb, wb = ctypes.c_size_t(), ctypes.c_size_t()
        assert lib.dllm_state_bytes(ctypes.byref(cfg), ctypes.byref(sb), ctypes.byref(wb)) == 0
        sizes.append((sb.value, wb.value))
    slab = run.batch * run.seq_len * m.d_model * 4
    extra = (m.n_layers - run.skip_layer - 1) * slab
    assert extra <= sizes[1][0] - sizes[0][0] <= extra + 4096
    assert sizes[1][1] == sizes[0][1]


def test_step_calls_reject_a_null_handle_without_a_gpu(lib):
    assert lib.dllm_begin_step(None, None, None) == 1
    assert lib.dllm_select_active(None, None, None, None, None) == 1
    assert lib.dllm_select_layers_forward(None, None, None) == 1
    assert lib.dllm_layers_forward(None, 0, 1, None) == 1
    assert lib.dllm_unmask(None, None, None, None, None) == 1

"""The allocation-free GEMM entry point (dllm_op_gemm_noalloc) against the regular one.

Callers that cannot allocate device memory (a framework that owns all of it and
hands over only inputs and outputs, or a hot path that must not call cudaMalloc)
use dllm_op_gemm_noalloc, whose scratch is a fixed array inside the library.
This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes when run on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _rowrel(a, b):
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    return float((np.abs(a - b).max(1) / np.maximum(np.abs(b).max(1), 1e-30)).max())


def _noalloc(lib, kind, W, X, out, count=None, rows_map=None):
    from token_skip_denoising_b200._lib import check, ptr, stream_ptr
    check(lib.dllm_op_gemm_noalloc(kind, ptr(W), W.shape[0], ptr(X), X.shape[0], ptr(count), W.shape[1], ptr(out),
                                   ptr(rows_map), stream_ptr()), "dllm_op_gemm_noalloc")


@pytest.fixture(scope="module")
def lib():
    from token_skip_denoising_b200 import _lib
    return _lib.load()


@pytest.mark.parametrize("rows,n_out,K", [(7, 384, 512), (32, 12288, 4096)])
def test_noalloc_matches_workspace_gemm_on_two_calls(lib, rows, n_out, K):
    from token_skip_denoising_b200 import ops
    g = torch.Generator(device=DEV).manual_seed(rows)
    for call in range(2):                                   # two calls in a row share the scratch
        W = (torch.randn((n_out, K), generator=g, device=DEV) * 0.05).to(torch.bfloat16)
        X = torch.randn((rows, K), generator=g, device=DEV).to(torch.bfloat16)
        ref = ops.gemm(W, X, kind=0)
        got = torch.full((rows, n_out), float("nan"), device=DEV)
        _noalloc(lib, 0, W, X, got)
        torch.cuda.synchronize()
        assert _rowrel(got.cpu().numpy(), ref.cpu().numpy()) < 1e-4, f"call {call}"
        # and the definition itself, X W^T in fp64 on the same bf16 operands
        exact = X.cpu().double().numpy() @ W.cpu().double().numpy().T
        assert _rowrel(got.cpu().numpy(), exact) < 1e-4, f"call {call}"


def test_noalloc_bf16_output_on_split_tiles(lib):
    """kind 1 (bf16 store) at the shape whose tiles are split across CTAs (12288 x 4096)."""
    from token_skip_denoising_b200 import ops
    g = torch.Generator(device=DEV).manual_seed(11)
    for call in range(2):
        W = (torch.randn((12288, 4096), generator=g, device=DEV) * 0.05).to(torch.bfloat16)
        X = torch.randn((32, 4096), generator=g, device=DEV).to(torch.bfloat16)
        ref = ops.gemm(W, X, kind=1)
        got = torch.zeros((32, 12288), dtype=torch.bfloat16, device=DEV)
        _noalloc(lib, 1, W, X, got)
        torch.cuda.synchronize()
        exact = X.cpu().double().numpy() @ W.cpu().double().numpy().T
        assert _rowrel(got.float().cpu().numpy(), ref.float().cpu().numpy()) < 2 ** -8, f"call {call}"
        assert _rowrel(got.float().cpu().numpy(), exact) < 2 ** -8, f"call {call}"


def test_noalloc_residual_with_device_count(lib):
    from token_skip_denoising_b200 import ops
    g = torch.Generator(device=DEV).manual_seed(7)
    W = (torch.randn((256, 1024), generator=g, device=DEV) * 0.05).to(torch.bfloat16)
    X = torch.randn((16, 1024), generator=g, device=DEV).to(torch.bfloat16)
    h0 = torch.randn((40, 256), generator=g, device=DEV)
    rmap = torch.tensor(list(range(3, 40, 3))[:16], dtype=torch.int32, device=DEV)
    cnt = torch.tensor([11], dtype=torch.int32, device=DEV)
    for _ in range(2):
        a, b = h0.clone(), h0.clone()
        ops.gemm(W, X, kind=3, out=a, rows_map=rmap, count=cnt)
        _noalloc(lib, 3, W, X, b, count=cnt, rows_map=rmap)
        torch.cuda.synchronize()
        assert _rowrel(b.cpu().numpy(), a.cpu().numpy()) < 1e-4


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    W = torch.zeros((256, 256), dtype=torch.bfloat16, device=DEV)
    X = torch.zeros((33, 256), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros((33, 256), device=DEV)
    from token_skip_denoising_b200._lib import ptr, stream_ptr
    rc = lib.dllm_op_gemm_noalloc(0, ptr(W), 256, ptr(X), 33, None, 256, ptr(out), None, stream_ptr())
    assert rc == 2
    assert b"at most 32 rows" in lib.dllm_last_error()

"""The allocation-free linear entry point (bat_linear_noalloc).

It serves callers that cannot call cudaMalloc and cannot obtain a device
workspace from their framework, for example a plugin running under an allocator
that already holds all device memory, or a serving loop that must not allocate
once it is running. It keeps the quantized activations in the library's own
static device scratch instead of a caller workspace. Its results must equal
those of bat_linear, the entry point that takes a workspace, bit for bit. Calls
in a row, with different inputs and a smaller call after a larger one, show that
stale scratch contents from an earlier call do not leak into the next one.

This file is collected last on purpose, so a failure here comes after every
other GPU test has run.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu

GEMM_TOL = 1e-3


def _dev_bf16(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def _dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def _rel(a: torch.Tensor, b: torch.Tensor) -> float:
    a64, b64 = a.double(), b.double()
    return (torch.linalg.norm(a64 - b64) / torch.linalg.norm(b64)).item()


def test_linear_noalloc_matches_linear_two_calls():
    import w4a4_bit_gemm_b200 as bat

    M, N, K = 300, 520, 1056
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=21)
    Ad, Bd, gl, gh = _dev_f32(A), _dev_f32(B), _dev_f32(g_lo), _dev_f32(g_hi)
    Wq = bat.bat_prepare_weight(_dev_bf16(wl.random_bf16((N, K), seed=22, scale=0.02)), Ad, Bd)
    for call, (seed, out_dtype) in enumerate([(23, torch.float32), (24, torch.bfloat16)]):
        X = _dev_bf16(wl.random_bf16((M, K), seed=seed, scale=1.0 + call))
        ref = bat.bat_linear(X, Wq, Ad, Bd, gl, gh, out_dtype=out_dtype)
        got = bat.bat_linear_noalloc(X, Wq, Ad, Bd, gl, gh, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert _rel(got.float(), ref.float()) <= GEMM_TOL, call
        # the same kernels on the same bytes: equal bit for bit
        assert torch.equal(got, ref), call
    assert bat.bat_device_error() == 0


def test_linear_noalloc_smaller_call_after_larger():
    """A large call leaves its codes and scales in the shared scratch; smaller ragged
    calls after it (rows inside the earlier call's 128-row groups, the tensor-core and
    the CUDA-core quantizer paths, K with padding blocks) must not see them."""
    import w4a4_bit_gemm_b200 as bat

    N, K = 264, 1056  # 33 blocks: the tiled scales carry padding blocks 33..35
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=41)
    Ad, Bd, gl, gh = _dev_f32(A), _dev_f32(B), _dev_f32(g_lo), _dev_f32(g_hi)
    Wq = bat.bat_prepare_weight(_dev_bf16(wl.random_bf16((N, K), seed=42, scale=0.02)), Ad, Bd)
    for i, M in enumerate([1000, 70, 5, 1000, 129]):
        X = _dev_bf16(wl.random_bf16((M, K), seed=43 + i, scale=1.0 + 3.0 * (i % 2)))
        ref = bat.bat_linear(X, Wq, Ad, Bd, gl, gh, out_dtype=torch.float32)
        got = bat.bat_linear_noalloc(X, Wq, Ad, Bd, gl, gh, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all(), M
        assert torch.equal(got, ref), M
    assert bat.bat_device_error() == 0


def test_linear_noalloc_rejects_oversize():
    import w4a4_bit_gemm_b200 as bat

    K = 4096
    M = bat.NOALLOC_SCRATCH_BYTES // (K // 2) + 1  # codes alone exceed the scratch
    assert bat.bat_linear_workspace_bytes(M, K) > bat.NOALLOC_SCRATCH_BYTES
    A, B, _, _ = wl.random_factors(K // 32, seed=3)
    Ad, Bd = _dev_f32(A), _dev_f32(B)
    Wq = bat.bat_prepare_weight(_dev_bf16(wl.random_bf16((64, K), seed=4, scale=0.02)), Ad, Bd)
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bat.BatError) as e:
        bat.bat_linear_noalloc(X, Wq, Ad, Bd)
    assert e.value.status == 7  # BAT_ERR_WORKSPACE

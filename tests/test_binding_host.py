"""The Python binding's own checks, on CPU: every tensor of a call on one device,
caller-supplied code/scale buffers large enough for the shape they claim, and the
right entry point reached with valid arguments.

The library is replaced by a recorder (size helpers still answer from libbat.so, which
is host code there); no compute entry point of the library is ever called, so these
tests are safe on any machine.
"""
from __future__ import annotations

import pytest
import torch

import w4a4_bit_gemm_b200 as bat


class _RecordingLib:
    SIZE = {"bat_mxfp4_codes_bytes", "bat_mxfp4_scales_bytes", "bat_mxfp8_codes_bytes",
            "bat_kv_codes_bytes", "bat_kv_scales_bytes", "bat_linear_workspace_bytes"}

    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in self.SIZE:
            return getattr(self.real, name)

        def record(*args):
            self.calls.append(name)
            return 0

        return record


@pytest.fixture
def rec(monkeypatch):
    r = _RecordingLib(bat.lib())
    monkeypatch.setattr(bat, "_lib", r)
    monkeypatch.setattr(bat, "_DEVICE_TYPE", "cpu")  # host tensors stand in for device ones
    monkeypatch.setattr(bat, "_stream", lambda s: None)
    return r


def _f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


def _bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def _factors(K, s=8):
    t = 32 // s
    return _f32(s, s), _f32(K // 32, t, t)


def test_valid_calls_reach_the_library(rec):
    M, N, K = 8, 16, 128
    A, B = _factors(K)
    g = _f32(K // 32)
    X, W = _bf16(M, K), _bf16(N, K)
    Xq = bat.bat_quantize_act(X, A, B, g, g)
    bat.bat_quantize_act_trace(X, A, B, g, g)
    Wq = bat.bat_prepare_weight(W, A, B)
    Y = bat.bat_mxfp4_gemm(Xq, Wq)
    assert Y.shape == (M, N) and Y.dtype == torch.bfloat16
    bat.bat_linear(X, Wq, A, B, g, g)
    bat.bat_linear_noalloc(X, Wq, A, B)
    A4, B4 = _factors(K, 4)
    bat.bat_quantize_act_gpk(X, A4, B4)
    bat.bat_prepare_weight_gpk(W, A4, B4)
    X8 = bat.bat_quantize_act_mxfp8(X, A, B, g, g)
    bat.bat_w4a8_gemm(X8, Wq, out_dtype=torch.float32)
    bat.bat_e2m1_encode(_f32(40))
    bat.bat_e4m3_encode(_f32(40))
    bat.bat_clip_ratios(g)
    cache = bat.KVCache.empty(6, 2, 64, "mxfp4", device="cpu")
    slots = torch.tensor([0, 3, -1], dtype=torch.int64)
    Ak, Bk = _factors(64)
    bat.bat_kv_quantize(_bf16(3, 2, 64), Ak, Bk, slots, cache)
    out = bat.bat_kv_dequantize(cache, slots)
    assert out.shape == (3, 2, 64)
    assert rec.calls == [
        "bat_quantize_act", "bat_quantize_act_trace", "bat_prepare_weight", "bat_mxfp4_gemm",
        "bat_linear", "bat_linear_noalloc", "bat_quantize_act_gpk", "bat_prepare_weight_gpk",
        "bat_quantize_act_mxfp8", "bat_w4a8_gemm", "bat_e2m1_encode", "bat_e4m3_encode",
        "bat_clip_ratios", "bat_kv_quantize", "bat_kv_dequantize"]


def test_linear_fused_flag_marshalled(monkeypatch):
    """bat_linear passes fused as the int argument before the stream (0 by default)."""
    seen = []

    class _Lib(_RecordingLib):
        def __getattr__(self, name):
            if name == "bat_linear":
                def rec_linear(*args):
                    seen.append(args)
                    return 0
                return rec_linear
            return super().__getattr__(name)

    monkeypatch.setattr(bat, "_lib", _Lib(bat.lib()))
    monkeypatch.setattr(bat, "_DEVICE_TYPE", "cpu")
    monkeypatch.setattr(bat, "_stream", lambda s: None)
    M, N, K = 8, 16, 128
    A, B = _factors(K)
    Wq = bat.MXFP4.empty(N, K, device="cpu")
    bat.bat_linear(_bf16(M, K), Wq, A, B)
    bat.bat_linear(_bf16(M, K), Wq, A, B, fused=True)
    assert len(seen) == 2
    assert len(seen[0]) == 13 and seen[0][11] == 0 and seen[1][11] == 1


def test_undersized_buffers_are_refused(rec):
    M, N, K = 8, 16, 64
    A, B = _factors(K)
    X = _bf16(M, K)
    small = bat.MXFP4.empty(4, K, device="cpu")
    # codes for 4 rows claimed as 8
    with pytest.raises(ValueError, match="codes"):
        bat.bat_quantize_act(X, A, B, Xq=bat.MXFP4(small.codes, small.scales, M, K))
    # enough codes, too few scale bytes (8 rows pad to 128, 2 blocks to 4: 512 bytes)
    codes = torch.empty(M * K // 2, dtype=torch.uint8)
    with pytest.raises(ValueError, match="scales"):
        bat.bat_quantize_act(X, A, B, Xq=bat.MXFP4(codes, small.scales[:256], M, K))
    # GEMM operands
    Xq = bat.bat_quantize_act(X, A, B)
    Wq = bat.MXFP4.empty(N, K, device="cpu")
    with pytest.raises(ValueError, match="Wq.codes"):
        bat.bat_mxfp4_gemm(Xq, bat.MXFP4(Wq.codes[:100], Wq.scales, N, K))
    # element conversion output, KV cache buffers
    with pytest.raises(ValueError, match="codes"):
        bat.bat_e2m1_encode(_f32(40), codes=torch.empty(39, dtype=torch.uint8))
    cache = bat.KVCache.empty(6, 2, 64, "mxfp8", device="cpu")
    short = bat.KVCache(cache.codes[:-1], cache.scales, 6, 2, 64, "mxfp8")
    Ak, Bk = _factors(64)
    with pytest.raises(ValueError, match="cache.codes"):
        bat.bat_kv_quantize(_bf16(3, 2, 64), Ak, Bk, torch.zeros(3, dtype=torch.int64), short)
    with pytest.raises(ValueError, match="cache.codes"):
        bat.bat_kv_dequantize(short, torch.zeros(3, dtype=torch.int64))
    assert rec.calls == ["bat_quantize_act"]  # only the valid quantize above got through


def test_mismatched_shapes_and_devices_are_refused(rec):
    K = 64
    A, B = _factors(K)
    Wq = bat.MXFP4.empty(16, 2 * K, device="cpu")
    with pytest.raises(ValueError, match="k=128"):
        bat.bat_linear(_bf16(8, K), Wq, A, B)
    with pytest.raises(ValueError, match="k=128"):
        bat.bat_linear_noalloc(_bf16(8, K), Wq, A, B)
    # a tensor somewhere else than the library's device type
    with pytest.raises(ValueError, match="CUDA"):
        bat.bat_quantize_act(_bf16(8, K), A, B.to("meta"))
    assert rec.calls == []


def test_host_tensors_are_refused_without_a_fake():
    """Unpatched: the binding refuses host tensors before touching the library."""
    A, B = _factors(64)
    with pytest.raises(ValueError, match="CUDA"):
        bat.bat_quantize_act(_bf16(4, 64), A, B)
    with pytest.raises(ValueError, match="CUDA"):
        bat.bat_e2m1_encode(_f32(8))

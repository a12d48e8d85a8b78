"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any CUDA call."""
from __future__ import annotations

import ctypes
import os

import pytest

import w4a4_bit_gemm_b200 as bat
from oracle import formats


@pytest.fixture(scope="module")
def L():
    from w4a4_bit_gemm_b200 import build
    build.build()
    return bat.lib()


def test_exports_every_declared_function(L):
    names = bat.declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_only_declared_functions_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", bat.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {n for n in exported if n.startswith("bat_")}
    assert ours == set(bat.declared_functions())


def test_sizes_match_documented_layout(L):
    for rows, k in [(1, 32), (64, 256), (130, 160), (2048, 4096), (16384, 4096), (6144, 4096)]:
        assert bat.bat_mxfp4_codes_bytes(rows, k) == rows * k // 2
        assert bat.bat_mxfp4_scales_bytes(rows, k) == formats.scale_bytes(rows, k // 32)
    assert bat.bat_mxfp4_codes_bytes(4, 48) == 0
    assert bat.bat_mxfp4_scales_bytes(0, 64) == 0
    assert bat.bat_linear_workspace_bytes(100, 64) == 3328 + formats.scale_bytes(100, 2)
    # decode sizes (<= 64 rows) and CTA-pair sizes (> 128 rows): codes and scales each
    # rounded to 256 bytes, then 4 KB of per-CTA completion flags for the two kernels
    up = lambda v: (v + 255) // 256 * 256
    for rows, k in [(16, 4096), (1, 32), (64, 12288), (300, 2048), (16384, 4096), (129, 4128)]:
        want = up(rows * k // 2) + up(formats.scale_bytes(rows, k // 32)) + 4096
        assert bat.bat_linear_workspace_bytes(rows, k) == want, (rows, k)


def test_status_strings(L):
    assert bat.bat_status_string(0) == "BAT_OK"
    assert bat.bat_status_string(4) == "BAT_ERR_SINGULAR"
    assert bat.bat_version() >= 100


def _fake_ptr(offset=0):
    return ctypes.c_void_p(0x7F0000000000 + offset)


def test_host_validation_returns_before_cuda(L):
    S = bat.MXFP4Struct
    good = S(0x7F0000100000, 0x7F0000200000, 4, 64)
    p = _fake_ptr()
    # null X
    assert L.bat_quantize_act(None, 4, 64, p, p, None, None, ctypes.byref(good), None) == 1
    # K not a multiple of 32
    g48 = S(0x7F0000100000, 0x7F0000200000, 4, 48)
    assert L.bat_quantize_act(p, 4, 48, p, p, None, None, ctypes.byref(g48), None) == 2
    # only one of the clip logits
    assert L.bat_quantize_act(p, 4, 64, p, p, p, None, ctypes.byref(good), None) == 1
    # output shape disagrees with X
    bad_rows = S(0x7F0000100000, 0x7F0000200000, 5, 64)
    assert L.bat_quantize_act(p, 4, 64, p, p, None, None, ctypes.byref(bad_rows), None) == 2
    # misaligned X
    assert L.bat_quantize_act(_fake_ptr(2), 4, 64, p, p, None, None, ctypes.byref(good), None) == 3
    # GEMM: K mismatch, bad dtype enum, misaligned Y
    w = S(0x7F0000300000, 0x7F0000400000, 8, 96)
    assert L.bat_mxfp4_gemm(ctypes.byref(good), ctypes.byref(w), p, 0, None) == 2
    w64 = S(0x7F0000300000, 0x7F0000400000, 8, 64)
    assert L.bat_mxfp4_gemm(ctypes.byref(good), ctypes.byref(w64), p, 7, None) == 1
    assert L.bat_mxfp4_gemm(ctypes.byref(good), ctypes.byref(w64), _fake_ptr(4), 0, None) == 3
    # linear: workspace too small or missing
    assert L.bat_linear(p, 4, ctypes.byref(w64), p, p, None, None, p, 0, None, 0, 0, None) == 7
    assert L.bat_linear(p, 4, ctypes.byref(w64), p, p, None, None, p, 0, p, 16, 0, None) == 7
    # linear: the fused flag is 0 or 1
    assert L.bat_linear(p, 4, ctypes.byref(w64), p, p, None, None, p, 0, p, 1 << 20, 2, None) == 1
    # weight prep: K too large / invalid N
    w_big = S(0x7F0000300000, 0x7F0000400000, 8, 262144 + 32)
    assert L.bat_prepare_weight(p, 8, 262144 + 32, p, p, None, None, ctypes.byref(w_big), None, None) == 2
    assert L.bat_prepare_weight(p, 0, 64, p, p, None, None, ctypes.byref(w64), None, None) == 1
    # element conversion / ratios: bad sizes
    assert L.bat_e2m1_encode(p, 0, p, None) == 1
    assert L.bat_clip_ratios(p, 0, p, None) == 1


def test_gpk_host_validation(L):
    S = bat.MXFP4Struct
    good = S(0x7F0000100000, 0x7F0000200000, 4, 64)
    p = _fake_ptr()
    # unsupported shared sizes are rejected before anything else
    for s in (0, 3, 5, 64, -8):
        assert L.bat_quantize_act_gpk(p, 4, 64, p, s, p, None, None, ctypes.byref(good), None,
                                      None) == 6
        assert L.bat_prepare_weight_gpk(p, 4, 64, p, s, p, None, None, ctypes.byref(good), None,
                                        None) == 6
    assert L.bat_quantize_act_gpk(None, 4, 64, p, 4, p, None, None, ctypes.byref(good), None,
                                  None) == 1
    assert L.bat_quantize_act_gpk(p, 4, 64, p, 4, p, None, None, ctypes.byref(good), _fake_ptr(4),
                                  None) == 3


def test_block_hadamard_factors_host():
    """Host-only helper: H_s/sqrt(s) and H_t/sqrt(t) in Sylvester order (scipy's)."""
    import numpy as np
    import scipy.linalg
    for s in (1, 2, 4, 8, 16, 32):
        A, B = bat.bat_block_hadamard_factors(s, 3)
        t = 32 // s
        assert np.array_equal(A.numpy(), (scipy.linalg.hadamard(s) / np.sqrt(s)).astype(np.float32))
        for b in range(3):
            assert np.array_equal(B[b].numpy(),
                                  (scipy.linalg.hadamard(t) / np.sqrt(t)).astype(np.float32))
    with pytest.raises(bat.BatError):
        bat.bat_block_hadamard_factors(3, 2)


def test_kv_and_w4a8_host_validation(L):
    p = _fake_ptr()
    # cache sizes
    assert bat.lib().bat_kv_codes_bytes(10, 8, 128, 0) == 10 * 8 * 128
    assert bat.lib().bat_kv_codes_bytes(10, 8, 128, 1) == 10 * 8 * 64
    assert bat.lib().bat_kv_scales_bytes(10, 8, 128) == 10 * 8 * 4
    assert bat.lib().bat_kv_codes_bytes(10, 8, 100, 0) == 0
    assert bat.lib().bat_mxfp8_codes_bytes(4, 64) == 256
    # kv store: bad split, bad head size, null pointers, bad format, misaligned slots
    args = lambda **kw: [kw.get("kv", p), kw.get("T", 4), kw.get("H", 2), kw.get("D", 64), p,
                         kw.get("s", 8), p, None, None, kw.get("slots", p), kw.get("fmt", 0), p, p,
                         kw.get("S", 8), None, None]
    assert L.bat_kv_quantize(*args(s=3)) == 6
    assert L.bat_kv_quantize(*args(D=48)) == 2
    assert L.bat_kv_quantize(*args(D=512)) == 2
    assert L.bat_kv_quantize(*args(kv=None)) == 1
    assert L.bat_kv_quantize(*args(fmt=7)) == 1
    assert L.bat_kv_quantize(*args(T=0)) == 1
    assert L.bat_kv_quantize(*args(slots=_fake_ptr(4))) == 3
    assert L.bat_kv_dequantize(p, p, 8, 2, 64, 0, p, 4, None, 8, None, p, 7, None) == 1
    assert L.bat_kv_dequantize(p, p, 8, 2, 64, 0, p, 4, p, 8, None, p, 0, None) == 1
    # W4A8 GEMM: K % 128 != 0, misaligned weight codes
    S = bat.MXFP4Struct
    x8 = S(0x7F0000100000, 0x7F0000200000, 4, 96)
    w8 = S(0x7F0000300000, 0x7F0000400000, 8, 96)
    assert L.bat_w4a8_gemm(ctypes.byref(x8), ctypes.byref(w8), p, 0, None) == 2
    x8 = S(0x7F0000100000, 0x7F0000200000, 4, 128)
    w8 = S(0x7F0000300010, 0x7F0000400000, 8, 128)
    assert L.bat_w4a8_gemm(ctypes.byref(x8), ctypes.byref(w8), p, 0, None) == 3


def test_row_limit(L):
    """Operands of more than 2^30 rows are rejected before any CUDA call: the tensor-memory
    copies address tiles by 32-bit signed coordinates."""
    S = bat.MXFP4Struct
    p = _fake_ptr()
    big = 1 << 30
    over = S(0x7F0000100000, 0x7F0000200000, big + 1, 64)
    w64 = S(0x7F0000300000, 0x7F0000400000, 8, 64)
    assert L.bat_quantize_act(p, big + 1, 64, p, p, None, None, ctypes.byref(over), None) == 2
    assert L.bat_mxfp4_gemm(ctypes.byref(over), ctypes.byref(w64), p, 0, None) == 2
    assert L.bat_mxfp4_gemm(ctypes.byref(w64), ctypes.byref(over), p, 0, None) == 2
    assert L.bat_prepare_weight(p, big + 1, 64, p, p, None, None, ctypes.byref(over), None,
                                None) == 2
    assert L.bat_linear(p, big + 1, ctypes.byref(w64), p, p, None, None, p, 0, p, 1 << 40,
                        0, None) == 2
    assert L.bat_linear_noalloc(p, big + 1, ctypes.byref(w64), p, p, None, None, p, 0, None) == 2
    # KV stores: tokens x heads, and cache slots x heads
    kv = lambda T, H, slots: L.bat_kv_quantize(p, T, H, 64, p, 8, p, None, None, p, 0, p, p,
                                               slots, None, None)
    assert kv(big // 2 + 1, 2, 8) == 2
    assert kv(4, 2, big // 2 + 1) == 2
    assert kv(4, big + 1, 8) == 2
    # exactly 2^30 rows passes the shape check: a misaligned X is what fails next
    at = S(0x7F0000100000, 0x7F0000200000, big, 64)
    assert L.bat_quantize_act(_fake_ptr(2), big, 64, p, p, None, None, ctypes.byref(at), None) == 3


def test_missing_library_fails_loudly():
    """The product path has no fallback: without libbat.so every call raises."""
    import subprocess
    import sys
    code = (
        "import w4a4_bit_gemm_b200 as bat\n"
        "bat.LIB_PATH = '/nonexistent/libbat.so'\n"
        "bat._lib = None\n"
        "try:\n"
        "    bat.bat_version()\n"
        "except RuntimeError as e:\n"
        "    print('raised', 'missing' in str(e))\n"
        "else:\n"
        "    print('no error')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    assert out.stdout.strip() == "raised True", out.stdout + out.stderr

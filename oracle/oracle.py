"""numpy front end of the C oracle (see ``bat_oracle.c`` for the readings).

Conventions: bf16 tensors are uint16 bit patterns; codes are one E2M1 code per
byte (unpacked, sign in bit 3); scales are plain row-major ``[rows][K/32]``
UE8M0 bytes (value 2**(byte-127)).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

G = 32
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
# element formats of the quantizer (the C side's ORC_E2M1 / ORC_E4M3)
FORMATS = {"e2m1": 0, "e4m3": 1}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.orc_transform_f64.argtypes = [P, I64, I64, P, P, P]
        L.orc_transform.argtypes = [P, I64, I64, P, P, P]
        L.orc_clip_ratio.argtypes = [ctypes.c_float]
        L.orc_clip_ratio.restype = ctypes.c_float
        L.orc_clip_ratios.argtypes = [P, I64, P]
        L.orc_e2m1_encode.argtypes = [ctypes.c_float]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_e2m1_encode_array.argtypes = [P, I64, P]
        L.orc_quantize_matrix.argtypes = [P, I64, I64, P, P, ctypes.c_int, P, P]
        L.orc_quantize_matrix.restype = I64
        L.orc_dequantize.argtypes = [P, P, I64, I64, P]
        L.orc_gemm_sampled.argtypes = [P, P, I64, P, I64, P, I64, P]
        L.orc_inverse.argtypes = [ctypes.c_int, P, P]
        L.orc_inverse.restype = ctypes.c_int
        L.orc_weight_transform_f64.argtypes = [P, I64, I64, P, P, P]
        L.orc_weight_transform_f64.restype = ctypes.c_int
        L.orc_kron.argtypes = [P, P, P]
        L.orc_kron_gen.argtypes = [P, P, ctypes.c_int, P]
        L.orc_transform_f64_gen.argtypes = [P, I64, I64, P, ctypes.c_int, P, P]
        L.orc_transform_gen.argtypes = [P, I64, I64, P, ctypes.c_int, P, P]
        L.orc_weight_transform_f64_gen.argtypes = [P, I64, I64, P, ctypes.c_int, P, P]
        L.orc_weight_transform_f64_gen.restype = ctypes.c_int
        L.orc_transform_vals_f64.argtypes = [P, I64, I64, P, ctypes.c_int, P, P]
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [ctypes.c_int]
        L.orc_e4m3_encode_array.argtypes = [P, I64, P]
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_quantize_matrix_fmt.argtypes = [P, I64, I64, P, P, ctypes.c_int, ctypes.c_int, P, P]
        L.orc_quantize_matrix_fmt.restype = I64
        L.orc_dequantize_fmt.argtypes = [P, P, I64, I64, ctypes.c_int, P]
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


SHARED_SIZES = (1, 2, 4, 8, 16, 32)


def factor_sizes(A: np.ndarray, B: np.ndarray, K: Optional[int] = None) -> int:
    """Shared size s of an (s x s) A with (K/32, 32/s, 32/s) private factors B."""
    s = int(np.shape(A)[0])
    if s not in SHARED_SIZES or np.shape(A) != (s, s):
        raise ValueError(f"shared factor must be s x s with s in {SHARED_SIZES}")
    t = G // s
    nb = np.shape(B)[0] if K is None else K // G
    if np.shape(B) != (nb, t, t):
        raise ValueError(f"private factors must be ({nb}, {t}, {t})")
    return s


def kron_block(B: np.ndarray, A: np.ndarray) -> np.ndarray:
    """The explicit 32x32 block P_b = B_b (x) A, fp64 (A is s x s, B_b (32/s) x (32/s))."""
    B = _c(B, np.float64)
    A = _c(A, np.float64)
    s = factor_sizes(A, B[None])
    P = np.empty((32, 32), np.float64)
    lib().orc_kron_gen(_p(B), _p(A), s, _p(P))
    return P


def transform_f64(X: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """x . P_b for every row and 32-element block; fp64, unrounded."""
    X = _c(X, np.uint16)
    M, K = X.shape
    assert K % G == 0
    s = factor_sizes(A, B, K)
    Y = np.empty((M, K), np.float64)
    lib().orc_transform_f64_gen(_p(X), M, K, _p(_c(A, np.float32)), s,
                                _p(_c(B, np.float32)), _p(Y))
    return Y


def transform(X: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """The transformed values: fp64 product rounded once to fp32."""
    X = _c(X, np.uint16)
    M, K = X.shape
    assert K % G == 0
    s = factor_sizes(A, B, K)
    Y = np.empty((M, K), np.float32)
    lib().orc_transform_gen(_p(X), M, K, _p(_c(A, np.float32)), s,
                            _p(_c(B, np.float32)), _p(Y))
    return Y


def clip_ratios(gamma: Optional[np.ndarray], n: Optional[int] = None) -> np.ndarray:
    """sigma(gamma) in fp64 rounded to fp32; ``None`` means no clip (ratio 1)."""
    if gamma is None:
        return np.ones(n, np.float32)
    g = _c(gamma, np.float32)
    r = np.empty(g.shape, np.float32)
    lib().orc_clip_ratios(_p(g), g.size, _p(r))
    return r


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e2m1_encode_array(_p(v), v.size, _p(out))
    return out


def e2m1_value(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, np.uint8)
    mag = GRID[codes & 7]
    return np.where(codes & 8, -mag, mag)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def e4m3_value(codes: np.ndarray) -> np.ndarray:
    table = np.array([lib().orc_e4m3_value(c) for c in range(256)])
    return table[np.asarray(codes, np.uint8)]


def quantize(Y: np.ndarray, r_lo: Optional[np.ndarray], r_hi: Optional[np.ndarray],
             per_row: bool = False, fmt: str = "e2m1"):
    """Clip + MX-quantize fp32 transformed values (E2M1 = MXFP4, E4M3 = MXFP8).
    Returns (codes, scales, n_bad); codes one per byte."""
    Y = _c(Y, np.float32)
    rows, K = Y.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // G), np.uint8)
    rl = None if r_lo is None else _c(r_lo, np.float32)
    rh = None if r_hi is None else _c(r_hi, np.float32)
    bad = lib().orc_quantize_matrix_fmt(_p(Y), rows, K, _p(rl), _p(rh), int(per_row),
                                        FORMATS[fmt], _p(codes), _p(scales))
    return codes, scales, int(bad)


def quantize_act(X: np.ndarray, A: np.ndarray, B: np.ndarray, g_lo: Optional[np.ndarray],
                 g_hi: Optional[np.ndarray], fmt: str = "e2m1"):
    """The whole online activation path: transform, clip, MX quantize."""
    nb = X.shape[1] // G
    Y = transform(X, A, B)
    r_lo = clip_ratios(g_lo, nb)
    r_hi = clip_ratios(g_hi, nb)
    codes, scales, _ = quantize(Y, r_lo, r_hi, fmt=fmt)
    return Y, codes, scales


def inverse(Mtx: np.ndarray) -> np.ndarray:
    Mtx = _c(Mtx, np.float64)
    n = Mtx.shape[0]
    out = np.empty_like(Mtx)
    if lib().orc_inverse(n, _p(Mtx), _p(out)):
        raise np.linalg.LinAlgError("singular")
    return out


def weight_transform_f64(W: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    W = _c(W, np.uint16)
    N, K = W.shape
    s = factor_sizes(A, B, K)
    out = np.empty((N, K), np.float64)
    if lib().orc_weight_transform_f64_gen(_p(W), N, K, _p(_c(A, np.float32)), s,
                                          _p(_c(B, np.float32)), _p(out)):
        raise np.linalg.LinAlgError("singular factor")
    return out


def prepare_weight(W: np.ndarray, A: np.ndarray, B: np.ndarray,
                   gw_lo: Optional[np.ndarray] = None, gw_hi: Optional[np.ndarray] = None):
    """Offline weight side: W P^-T rounded to fp32, optional per-(row, block) clip, MXFP4."""
    N, K = W.shape
    Wt = weight_transform_f64(W, A, B).astype(np.float32)
    r_lo = None if gw_lo is None else clip_ratios(gw_lo.reshape(-1)).reshape(N, K // G)
    r_hi = None if gw_hi is None else clip_ratios(gw_hi.reshape(-1)).reshape(N, K // G)
    codes, scales, _ = quantize(Wt, r_lo, r_hi, per_row=True)
    return Wt, codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, fmt: str = "e2m1") -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    lib().orc_dequantize_fmt(_p(codes), _p(scales), rows, K, FORMATS[fmt], _p(out))
    return out


def gemm_sampled(Xd: np.ndarray, Wd: np.ndarray, rows: Optional[Sequence[int]] = None,
                 cols: Optional[Sequence[int]] = None) -> np.ndarray:
    """fp64 Y[rows][cols] = Xd Wd^T, one serial sum per output element."""
    Xd = _c(Xd, np.float64)
    Wd = _c(Wd, np.float64)
    K = Xd.shape[1]
    r = np.arange(Xd.shape[0], dtype=np.int64) if rows is None else _c(rows, np.int64)
    c = np.arange(Wd.shape[0], dtype=np.int64) if cols is None else _c(cols, np.int64)
    Y = np.empty((r.size, c.size), np.float64)
    lib().orc_gemm_sampled(_p(Xd), _p(Wd), K, _p(r), r.size, _p(c), c.size, _p(Y))
    return Y


def linear(X, W, A, B, g_lo, g_hi, rows=None, cols=None, act_fmt: str = "e2m1"):
    """Y = Q(XP) Q(P^-1 W^T) in fp64, optionally on a sample of outputs; activations
    in MXFP4 (W4A4) or MXFP8 E4M3 (W4A8), weights in MXFP4."""
    _, xc, xs = quantize_act(X, A, B, g_lo, g_hi, fmt=act_fmt)
    _, wc, ws = prepare_weight(W, A, B)
    return gemm_sampled(dequantize(xc, xs, act_fmt), dequantize(wc, ws), rows, cols)


def gpk_param_counts(K: int, shared: int = 8, private: int = 4) -> dict:
    """Transform parameter counts for hidden size K with g = shared*private."""
    g = shared * private
    nb = K // g
    return {
        "gpk": shared * shared + nb * private * private,
        "naive_kronecker": nb * (shared * shared + private * private),
        "full_blocks": nb * g * g,
    }


def num_threads() -> int:
    """Host threads the oracle's parallel loops use."""
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Thread count of the oracle's parallel loops (results do not depend on it)."""
    lib().orc_set_num_threads(int(n))


def transform_vals_f64(Xd: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """x . (B_b (x) A) for an fp64 matrix (any split); fp64, unrounded."""
    Xd = _c(Xd, np.float64)
    M, K = Xd.shape
    s = factor_sizes(A, B, K)
    Y = np.empty((M, K), np.float64)
    lib().orc_transform_vals_f64(_p(Xd), M, K, _p(_c(A, np.float32)), s, _p(_c(B, np.float32)),
                                 _p(Y))
    return Y


# ---------------------------------------------------------------- KV-cache path
# The note (Key Designs 4, "Equivalent Transformer integration") puts one transform
# set on the per-head key path and one on the value path, and the settings KV8 / KV4
# quantize the cache to MXFP8 (E4M3) / MXFP4. Reading: every head's D-vector
# (D = head_dim, a multiple of 32) is transformed by the same factors (A shared,
# B[D/32] one per 32-channel block of the head), clipped with per-block logits
# [D/32] shared by heads and tokens, quantized, and stored at the token's cache
# slot; slot -1 means "do not store".

def kv_quantize(kv: np.ndarray, A, B, g_lo, g_hi, fmt: str, slots, cache_codes, cache_scales):
    """kv: bf16 bits [T][H][D]; cache_codes [S][H][D] (one code per byte),
    cache_scales [S][H][D/32]; both updated in place at rows slots[t] >= 0.
    Returns the fp32 transformed values [T][H][D]."""
    T, H, D = kv.shape
    Y, codes, scales = quantize_act(kv.reshape(T * H, D), A, B, g_lo, g_hi, fmt=fmt)
    codes = codes.reshape(T, H, D)
    scales = scales.reshape(T, H, D // G)
    for t in range(T):
        if slots[t] >= 0:
            cache_codes[slots[t]] = codes[t]
            cache_scales[slots[t]] = scales[t]
    return Y.reshape(T, H, D)


def kv_dequantize(cache_codes, cache_scales, slots, fmt: str, A_out=None, B_out=None):
    """Values of the cache rows slots[t] ([T][H][D], fp64), optionally multiplied per
    32-block by B_out (x) A_out (the inverse factors give back the untransformed K/V)."""
    S, H, D = cache_codes.shape
    T = len(slots)
    c = np.asarray(cache_codes)[np.asarray(slots)].reshape(T * H, D)
    sc = np.asarray(cache_scales)[np.asarray(slots)].reshape(T * H, D // G)
    v = dequantize(c, sc, fmt)
    if A_out is not None:
        v = transform_vals_f64(v, A_out, B_out)
    return v.reshape(T, H, D)

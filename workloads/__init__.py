"""Seeded synthetic inputs for the BATQuant W4A4 linear layer.

This module only draws random numbers and packs them as bf16 bit patterns. It
holds none of the method's arithmetic, so both the CPU oracle and the CUDA path
can take their inputs from it without sharing any of the computation.

The recipe follows the layer shapes of the BATQuant note (en.papernotes.org,
"Equivalent Transformer integration": the transform sits before gate/up,
down_proj, qkv_proj and o_proj of Qwen3-8B-class models, hidden size 4096):

* ``A = I + 0.1 N(0,1)`` (8x8, shared by all blocks), ``B_b = I + 0.1 N(0,1)``
  (4x4, one per 32-channel block), clip logits ``gamma ~ U(1, 4)``.
* Outlier channels are picked without replacement and scaled column-wise.
* Draw order is fixed: X, outlier picks (and their factors), W, A, B, gamma_lo,
  gamma_hi, all from one ``numpy.random.Generator(PCG64(seed))``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

G = 32  # MXFP block size (elements per shared scale)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    K: int
    x_kind: str            # "normal", "silu_gate", "student_t"
    outlier_frac: float
    outlier_lo: float      # outlier factor range; lo == hi means a fixed factor
    outlier_hi: float
    description: str

    @property
    def nb(self) -> int:
        return self.K // G


WORKLOADS = {
    "tiny": Workload("tiny", 64, 128, 256, "normal", 0.02, 50.0, 50.0,
                     "X 64x256 N(0,1), 2% channels x50; W 128x256 N(0,0.02)"),
    "mlp_gate_up": Workload("mlp_gate_up", 2048, 24576, 4096, "normal", 0.01, 30.0, 100.0,
                            "Qwen3-8B-like MLP gate||up: X 2048x4096 N(0,1), 1% channels x U(30,100); "
                            "W 24576x4096 N(0,0.02)"),
    "mlp_down": Workload("mlp_down", 2048, 4096, 12288, "silu_gate", 0.005, 200.0, 200.0,
                         "MLP down_proj: X 2048x12288 = SiLU(g)*u, 0.5% channels x200; "
                         "W 4096x12288 N(0,0.02)"),
    "decode_qkv": Workload("decode_qkv", 16, 6144, 4096, "normal", 0.01, 30.0, 100.0,
                           "decode qkv_proj: X 16x4096 as mlp_gate_up; W 6144x4096 (q 4096|k 1024|v 1024)"),
    "prefill_o": Workload("prefill_o", 16384, 4096, 4096, "student_t", 0.01, 50.0, 50.0,
                          "long-prefill o_proj: X 16384x4096 Student-t(3)/sqrt(3), 1% channels x50; "
                          "W 4096x4096 N(0,0.02)"),
}
# Ordered as the layer list is usually quoted: tiny first, then the four layer shapes.
ORDER = ["tiny", "mlp_gate_up", "mlp_down", "decode_qkv", "prefill_o"]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) and return the 16-bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Inputs:
    X: np.ndarray        # uint16 bf16 bits [M][K]
    W: np.ndarray        # uint16 bf16 bits [N][K]
    A: np.ndarray        # float32 [8][8]
    B: np.ndarray        # float32 [nb][4][4]
    g_lo: np.ndarray     # float32 [nb]
    g_hi: np.ndarray     # float32 [nb]
    outlier_channels: np.ndarray


def _draw_x(rng: np.random.Generator, wl: Workload, M: int) -> tuple[np.ndarray, np.ndarray]:
    K = wl.K
    if wl.x_kind == "normal":
        x = rng.standard_normal((M, K), dtype=np.float32)
    elif wl.x_kind == "silu_gate":
        g = rng.standard_normal((M, K), dtype=np.float32)
        u = rng.standard_normal((M, K), dtype=np.float32)
        x = (g / (1.0 + np.exp(-g))) * u
    elif wl.x_kind == "student_t":
        x = (rng.standard_t(3.0, size=(M, K)) / np.sqrt(3.0)).astype(np.float32)
    else:
        raise ValueError(wl.x_kind)
    n_out = max(1, int(round(wl.outlier_frac * K)))
    chans = np.sort(rng.choice(K, size=n_out, replace=False))
    if wl.outlier_lo == wl.outlier_hi:
        fac = np.full(n_out, wl.outlier_lo, dtype=np.float32)
    else:
        fac = rng.uniform(wl.outlier_lo, wl.outlier_hi, size=n_out).astype(np.float32)
    x[:, chans] *= fac[None, :]
    return x.astype(np.float32), chans


def make_inputs(name: str, seed: int = 0, M: Optional[int] = None, N: Optional[int] = None,
                with_weight: bool = True) -> Inputs:
    """Draw one workload. ``M``/``N`` override the row counts (same recipe)."""
    wl = WORKLOADS[name]
    M = wl.M if M is None else M
    N = wl.N if N is None else N
    rng = np.random.Generator(np.random.PCG64(seed))
    x, chans = _draw_x(rng, wl, M)
    if with_weight:
        w = (0.02 * rng.standard_normal((N, wl.K), dtype=np.float32)).astype(np.float32)
    else:
        w = np.zeros((0, wl.K), dtype=np.float32)
    A = (np.eye(8) + 0.1 * rng.standard_normal((8, 8))).astype(np.float32)
    B = (np.eye(4)[None] + 0.1 * rng.standard_normal((wl.nb, 4, 4))).astype(np.float32)
    g_lo = rng.uniform(1.0, 4.0, size=wl.nb).astype(np.float32)
    g_hi = rng.uniform(1.0, 4.0, size=wl.nb).astype(np.float32)
    return Inputs(f32_to_bf16_bits(x), f32_to_bf16_bits(w), A, B, g_lo, g_hi, chans)


def random_factors(nb: int, seed: int, shared: int = 8
                   ) -> tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """A, B, gamma_lo, gamma_hi with the standard recipe, for ad-hoc shapes.

    ``shared`` is the size s of the shared factor A (s x s); the private
    factors are (32/s) x (32/s). An n x n factor is I + c N(0,1) with
    c = 0.1 min(1, sqrt(8/n)), so the 16 and 32 sizes stay as well conditioned
    as the default 8 and 4 ones; with s = 8 the draws are the default ones.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    t = 32 // shared
    ca = 0.1 * min(1.0, np.sqrt(8.0 / shared))
    cb = 0.1 * min(1.0, np.sqrt(8.0 / t))
    A = (np.eye(shared) + ca * rng.standard_normal((shared, shared))).astype(np.float32)
    B = (np.eye(t)[None] + cb * rng.standard_normal((nb, t, t))).astype(np.float32)
    g_lo = rng.uniform(1.0, 4.0, size=nb).astype(np.float32)
    g_hi = rng.uniform(1.0, 4.0, size=nb).astype(np.float32)
    return A, B, g_lo, g_hi


def random_bf16(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return f32_to_bf16_bits((scale * rng.standard_normal(shape)).astype(np.float32))

"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources are the pages (BATQuant note on en.papernotes.org, the nubint.ai review,
the BRQ article on 10100.com), closed forms, library routines (numpy/scipy),
brute force and exact rational arithmetic. Every test here runs on the CPU.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle
from oracle import formats
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_pairs(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            rows.append((a, b))
    return rows


def _bf16_to_f64(h):
    return wl.bf16_bits_to_f32(h).astype(np.float64)


# --- MXFP4 element grid and encoder -------------------------------------------------

def test_grid_matches_pages():
    """Code -> value table equals the grid the note prints (Background & Motivation)."""
    table = {int(a): float(b) for a, b in _read_pairs("e2m1_grid.txt")}
    codes = np.arange(16, dtype=np.uint8)
    vals = oracle.e2m1_value(codes)
    for c in range(8):
        assert vals[c] == table[c]
        assert vals[c + 8] == -table[c]


def test_e2m1_ties_fixture():
    for v, code in _read_pairs("e2m1_ties.txt"):
        assert oracle.e2m1_encode(np.array([np.float32(v)]))[0] == int(code), v


def _e2m1_by_binade(v: np.ndarray) -> np.ndarray:
    """E2M1 as a 1-mantissa-bit float: round-half-even on each binade's step.

    Below 2 the step is 0.5 (subnormal code range and the [1, 2) binade),
    on [2, 4) it is 1, on [4, 8) it is 2; anything above 6 saturates. This is
    textbook IEEE-style rounding with numpy's rint (ties to even), a different
    formulation from the oracle's nearest-point search.
    """
    a = np.abs(v.astype(np.float64))
    q = np.where(a < 2.0, np.rint(a * 2.0) / 2.0,
                 np.where(a < 4.0, np.rint(a), 2.0 * np.rint(a / 2.0)))
    q = np.minimum(q, 6.0)
    lut = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    keys = np.array(sorted(lut))
    code = np.searchsorted(keys, q).astype(np.uint8)
    assert np.all(keys[code] == q)
    return code | (np.signbit(v).astype(np.uint8) << 3)


def test_e2m1_bruteforce_all_fp32_up_to_8():
    """Every fp32 bit pattern in [0, 8] (about 1.09e9 values), plus sampled negatives."""
    top = np.float32(8.0).view(np.uint32)
    step = 1 << 26
    for start in range(0, int(top) + 1, step):
        bits = np.arange(start, min(start + step, int(top) + 1), dtype=np.uint32)
        v = bits.view(np.float32)
        got = oracle.e2m1_encode(v)
        want = _e2m1_by_binade(v)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])
    rng = np.random.default_rng(1)
    bits = rng.integers(0, int(top) + 1, size=2_000_000, dtype=np.uint32) | np.uint32(0x80000000)
    v = bits.view(np.float32)
    assert np.array_equal(oracle.e2m1_encode(v), _e2m1_by_binade(v))


# --- GPK structure ----------------------------------------------------------------

def test_param_counts_printed():
    g = dict(_read_pairs("gpk_param_counts.txt"))
    counts = oracle.gpk_param_counts(int(g["hidden"]))
    assert counts["gpk"] == int(g["gpk"])
    assert counts["naive_kronecker"] == int(g["naive_kronecker"])
    assert counts["full_blocks"] == int(g["full_blocks"])
    # the review's ">74%-79%" reduction claim
    assert 100 * (1 - counts["gpk"] / int(g["flatquant"])) > int(g["reduction_vs_flatquant_min_pct"])
    assert 100 * (1 - counts["gpk"] / counts["naive_kronecker"]) > int(g["reduction_vs_naive_min_pct"])


def test_kron_block_equals_numpy_kron():
    A, B, _, _ = wl.random_factors(3, seed=5)
    for b in range(3):
        P = oracle.kron_block(B[b], A)
        assert np.array_equal(P, np.kron(B[b].astype(np.float64), A.astype(np.float64)))


def test_transform_equals_block_diagonal_matmul():
    """x P with P = blockdiag(B_b (x) A) built by scipy, and the factored form."""
    inp = wl.make_inputs("tiny")
    nb = inp.B.shape[0]
    P = scipy.linalg.block_diag(*[np.kron(inp.B[b].astype(np.float64), inp.A.astype(np.float64))
                                  for b in range(nb)])
    X = _bf16_to_f64(inp.X)
    Y = oracle.transform_f64(inp.X, inp.A, inp.B)
    ref = X @ P
    assert np.max(np.abs(Y - ref)) <= 1e-14 * np.max(np.abs(ref))
    # factored form vec_row(B_b^T X_r A), X_r[i][p] = x[8i+p]
    A64 = inp.A.astype(np.float64)
    for b in range(nb):
        Xr = X[:, 32 * b:32 * b + 32].reshape(-1, 4, 8)
        fac = (inp.B[b].astype(np.float64).T[None] @ Xr @ A64[None]).reshape(-1, 32)
        blk = Y[:, 32 * b:32 * b + 32]
        assert np.max(np.abs(blk - fac)) <= 1e-14 * np.max(np.abs(fac))
    # the fp32 transformed values are that product rounded once
    assert np.array_equal(oracle.transform(inp.X, inp.A, inp.B), Y.astype(np.float32))


def test_block_locality():
    """Changing block b of x changes only block b's transform, codes and scale."""
    inp = wl.make_inputs("tiny")
    X = inp.X.copy()
    Y0, c0, s0 = oracle.quantize_act(X, inp.A, inp.B, inp.g_lo, inp.g_hi)
    b = 3
    X[:, 32 * b:32 * b + 32] = wl.random_bf16((X.shape[0], 32), seed=9, scale=20.0)
    Y1, c1, s1 = oracle.quantize_act(X, inp.A, inp.B, inp.g_lo, inp.g_hi)
    other = np.ones(X.shape[1], bool)
    other[32 * b:32 * b + 32] = False
    assert np.array_equal(Y0[:, other], Y1[:, other])
    assert np.array_equal(c0[:, other], c1[:, other])
    keep = np.arange(s0.shape[1]) != b
    assert np.array_equal(s0[:, keep], s1[:, keep])
    assert not np.array_equal(Y0[:, ~other], Y1[:, ~other])


# --- inverse and weight-side fusion -------------------------------------------------

def test_inverse_roundtrip_and_library():
    rng = np.random.default_rng(3)
    for n in (1, 2, 4, 8, 16, 32):
        for _ in range(20):
            M = np.eye(n) + 0.3 * min(1.0, np.sqrt(8.0 / n)) * rng.standard_normal((n, n))
            inv = oracle.inverse(M)
            assert np.max(np.abs(inv @ M - np.eye(n))) < 1e-12
            assert np.allclose(inv, np.linalg.inv(M), rtol=1e-12, atol=1e-12)
    with pytest.raises(np.linalg.LinAlgError):
        oracle.inverse(np.zeros((4, 4)))


def test_inverse_fusion_preserves_output():
    """(X P)(P^-1 W^T) = X W^T before quantization (Key Designs 1)."""
    inp = wl.make_inputs("tiny")
    XP = oracle.transform_f64(inp.X, inp.A, inp.B)
    WPt = oracle.weight_transform_f64(inp.W, inp.A, inp.B)
    ref = _bf16_to_f64(inp.X) @ _bf16_to_f64(inp.W).T
    got = XP @ WPt.T
    assert np.linalg.norm(got - ref) <= 1e-10 * np.linalg.norm(ref)


def test_hadamard_special_case():
    """A = H8/sqrt8, B_b = H4/2 gives P_b = H32/sqrt32 (Sylvester), the block rotation of BRQ."""
    H8 = scipy.linalg.hadamard(8) / np.sqrt(8.0)
    H4 = scipy.linalg.hadamard(4) / 2.0
    H32 = scipy.linalg.hadamard(32) / np.sqrt(32.0)
    A = H8.astype(np.float32)
    nb = 8
    B = np.repeat(H4[None].astype(np.float32), nb, axis=0)
    assert np.allclose(oracle.kron_block(B[0], A), H32, atol=1e-7)
    X = wl.random_bf16((16, 32 * nb), seed=11)
    Y = oracle.transform_f64(X, A, B)
    Xd = _bf16_to_f64(X)
    n_in = np.linalg.norm(Xd.reshape(16, nb, 32), axis=2)
    n_out = np.linalg.norm(Y.reshape(16, nb, 32), axis=2)
    assert np.allclose(n_in, n_out, rtol=1e-6)
    # orthonormal and symmetric, so P^-T = P: the weight side equals the activation side
    assert np.allclose(oracle.weight_transform_f64(X, A, B), Y, rtol=1e-6, atol=1e-6)


# --- quantizer ----------------------------------------------------------------------

def _rtn_mxfp4(x: np.ndarray):
    """Plain MXFP4 round-to-nearest of a matrix, written independently of the oracle."""
    rows, K = x.shape
    blocks = x.reshape(rows, K // 32, 32).astype(np.float32)
    amax = np.max(np.abs(blocks), axis=2)
    with np.errstate(divide="ignore"):
        e = np.where(amax > 0, np.floor(np.log2(amax.astype(np.float64))) - 2, -127)
    e = np.clip(e, -127, 127).astype(np.int32)
    v = blocks.astype(np.float64) / np.exp2(e.astype(np.float64))[..., None]
    v = np.where(v == 0, 0.0, v)  # exact zeros become +0
    codes = _e2m1_by_binade(v.astype(np.float32)).reshape(rows, K)
    return codes, (e + 127).astype(np.uint8)


def test_rtn_special_case():
    """Identity factors with no clip reduce to plain MXFP4 RTN (the RTN row of Table 2)."""
    inp = wl.make_inputs("tiny")
    nb = inp.B.shape[0]
    A = np.eye(8, dtype=np.float32)
    B = np.repeat(np.eye(4, dtype=np.float32)[None], nb, axis=0)
    Y, codes, scales = oracle.quantize_act(inp.X, A, B, None, None)
    x = wl.bf16_bits_to_f32(inp.X)
    assert np.array_equal(Y, x)
    rc, rs = _rtn_mxfp4(x)
    assert np.array_equal(scales, rs)
    assert np.array_equal(codes, rc)
    # gamma = +inf is the same as "no clip" (ratio exactly 1)
    inf = np.full(nb, np.inf, np.float32)
    _, c2, s2 = oracle.quantize_act(inp.X, A, B, inf, inf)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)


@pytest.mark.parametrize("name", ["tiny"])
def test_grid_and_scale_rule(name):
    inp = wl.make_inputs(name)
    Y, codes, scales = oracle.quantize_act(inp.X, inp.A, inp.B, inp.g_lo, inp.g_hi)
    deq = oracle.dequantize(codes, scales)
    rows, K = codes.shape
    e = scales.astype(np.int64) - 127
    assert np.all(scales < 255)
    mant = deq.reshape(rows, K // 32, 32) / np.exp2(e)[..., None]
    assert np.all(np.isin(np.abs(mant), oracle.GRID))
    # the block maximum lands on 4 or 6: amax * 2^-e in [4, 8) for every non-zero block
    nz = np.any(codes.reshape(rows, K // 32, 32) & 7, axis=2)
    top = np.max(np.abs(mant), axis=2)
    assert np.all(np.isin(top[nz], [4.0, 6.0]))
    r_lo = oracle.clip_ratios(inp.g_lo)
    r_hi = oracle.clip_ratios(inp.g_hi)
    blk = Y.reshape(rows, K // 32, 32)
    lo = (r_lo[None] * blk.min(axis=2)).astype(np.float32)
    hi = (r_hi[None] * blk.max(axis=2)).astype(np.float32)
    c = np.minimum(np.maximum(blk, lo[..., None]), hi[..., None])
    amax = np.max(np.abs(c), axis=2).astype(np.float64)
    ratio = amax[nz] / np.exp2(e[nz])
    assert np.all((ratio >= 4.0) & (ratio < 8.0))


def test_clip_properties():
    rng = np.random.default_rng(7)
    Y = (rng.standard_normal((50, 64)) * rng.uniform(0.1, 50, size=(50, 1))).astype(np.float32)
    Y[0, :32] = np.abs(Y[0, :32]) + 1.0          # all-positive block: lower bound inert
    Y[1, 32:] = -np.abs(Y[1, 32:]) - 1.0         # all-negative block: upper bound inert
    r_lo = np.array([0.7, 0.9], np.float32)
    r_hi = np.array([0.8, 0.6], np.float32)
    codes, scales, bad = oracle.quantize(Y, r_lo, r_hi)
    assert bad == 0
    # no clip when both ratios are 1
    c1, s1, _ = oracle.quantize(Y, np.ones(2, np.float32), np.ones(2, np.float32))
    c0, s0, _ = oracle.quantize(Y, None, None)
    assert np.array_equal(c1, c0) and np.array_equal(s1, s0)
    blk = Y.reshape(50, 2, 32)
    lo = (r_lo[None] * blk.min(axis=2)).astype(np.float32)
    hi = (r_hi[None] * blk.max(axis=2)).astype(np.float32)
    clipped = np.clip(blk, lo[..., None], hi[..., None])
    amax = np.abs(clipped).max(axis=2)
    assert np.all(amax <= np.maximum(np.abs(lo), np.abs(hi)))
    # the quantized block equals RTN of the numpy-clipped values (hi wins if lo > hi)
    rc, rs = _rtn_mxfp4(np.minimum(np.maximum(blk, lo[..., None]), hi[..., None]).reshape(50, 64))
    assert np.array_equal(codes, rc) and np.array_equal(scales, rs)
    # bounds are inert on one-signed blocks
    assert lo[0, 0] <= blk[0, 0].min() and hi[1, 1] >= blk[1, 1].max()


def test_weight_clip_per_row_and_block():
    """Weight clip (the note, Key Designs 3: weights receive the analogous treatment):
    one logit pair per (output row, block), written independently here with scipy's
    logistic, a numpy clamp and the separately written RTN quantizer."""
    inp = wl.make_inputs("tiny")
    N, K = inp.W.shape
    nb = K // 32
    assert N != nb  # a transposed [block][row] index cannot line up by accident
    rng = np.random.default_rng(31)
    gw_lo = rng.uniform(-1.0, 3.0, size=(N, nb)).astype(np.float32)
    gw_hi = rng.uniform(-1.0, 3.0, size=(N, nb)).astype(np.float32)
    Wt, codes, scales = oracle.prepare_weight(inp.W, inp.A, inp.B, gw_lo, gw_hi)
    # the transformed weights themselves are unclipped (pinned by inverse fusion)
    assert np.array_equal(Wt, oracle.weight_transform_f64(inp.W, inp.A, inp.B).astype(np.float32))

    def rtn_with(r_lo, r_hi):
        blk = Wt.reshape(N, nb, 32)
        lo = (r_lo * blk.min(axis=2)).astype(np.float32)
        hi = (r_hi * blk.max(axis=2)).astype(np.float32)
        c = np.minimum(np.maximum(blk, lo[..., None]), hi[..., None])
        return _rtn_mxfp4(c.reshape(N, K))

    r_lo = scipy.special.expit(gw_lo.astype(np.float64)).astype(np.float32)
    r_hi = scipy.special.expit(gw_hi.astype(np.float64)).astype(np.float32)
    rc, rs = rtn_with(r_lo, r_hi)
    assert np.array_equal(codes, rc) and np.array_equal(scales, rs)
    # the quantizer's per-row branch alone, fed the same ratios
    qc, qs, bad = oracle.quantize(Wt, r_lo, r_hi, per_row=True)
    assert bad == 0 and np.array_equal(qc, rc) and np.array_equal(qs, rs)
    # controls: the plausible index mistakes give other codes, so this test would see them
    flat_lo, flat_hi = r_lo.reshape(-1), r_hi.reshape(-1)
    transposed = rtn_with(flat_lo.reshape(nb, N).T, flat_hi.reshape(nb, N).T)  # b * N + m
    shared = rtn_with(np.broadcast_to(flat_lo[:nb], (N, nb)), np.broadcast_to(flat_hi[:nb], (N, nb)))
    for wc, ws in (transposed, shared):
        assert not (np.array_equal(wc, codes) and np.array_equal(ws, scales))
    # the clip is active: most (row, block) pairs change against the unclipped weights
    _, uc, _ = oracle.prepare_weight(inp.W, inp.A, inp.B)
    changed = np.any((uc != codes).reshape(N, nb, 32), axis=2)
    assert changed.mean() > 0.5


def test_sigmoid_ratios():
    g = np.array([0.0, 1.0, 2.5, 4.0, -3.0, 30.0], np.float32)
    r = oracle.clip_ratios(g)
    assert r[0] == np.float32(0.5)
    assert np.array_equal(r, scipy.special.expit(g.astype(np.float64)).astype(np.float32))
    assert oracle.clip_ratios(np.array([np.inf], np.float32))[0] == 1.0
    assert np.all(oracle.clip_ratios(None, 4) == 1.0)


def test_zero_and_degenerate_blocks():
    Y = np.zeros((2, 64), np.float32)
    Y[1, :] = -0.0
    Y[1, 40] = 3.0
    codes, scales, _ = oracle.quantize(Y, None, None)
    assert np.all(scales[0] == 0) and np.all(codes[0] == 0)   # amax = 0: e = -127, byte 0
    assert scales[1, 0] == 0 and np.all(codes[1, :32] == 0)   # -0 encodes as +0
    # 3.0: floor(log2 3) - 2 = -1, byte 126, 3 * 2 = 6 -> code 7
    assert scales[1, 1] == 126 and codes[1, 40] == 7
    # non-finite input is flagged
    Y2 = np.zeros((1, 32), np.float32)
    Y2[0, 5] = np.inf
    _, s2, bad = oracle.quantize(Y2, None, None)
    assert bad == 1 and s2[0, 0] == 0xFF


# --- GEMM ---------------------------------------------------------------------------

def test_dequantize_closed_form():
    codes = np.array([[7, 15, 1, 9] * 8], np.uint8)
    scales = np.array([[127 + 3]], np.uint8)
    d = oracle.dequantize(codes, scales)
    assert np.array_equal(d[0, :4], np.array([6.0, -6.0, 0.5, -0.5]) * 8.0)


def test_gemm_exact_rational():
    """fp64 dot products of dequantized MXFP4 operands against exact Fractions."""
    inp = wl.make_inputs("tiny")
    _, xc, xs = oracle.quantize_act(inp.X, inp.A, inp.B, inp.g_lo, inp.g_hi)
    _, wc, ws = oracle.prepare_weight(inp.W, inp.A, inp.B)
    Xd = oracle.dequantize(xc, xs)
    Wd = oracle.dequantize(wc, ws)
    rows = [0, 17, 63]
    cols = [0, 5, 64, 127]
    Y = oracle.gemm_sampled(Xd, Wd, rows, cols)
    K = Xd.shape[1]
    for i, m in enumerate(rows):
        for j, n in enumerate(cols):
            exact = Fraction(0)
            mag = Fraction(0)
            for k in range(K):
                t = Fraction(Xd[m, k]) * Fraction(Wd[n, k])
                exact += t
                mag += abs(t)
            assert abs(Fraction(Y[i, j]) - exact) <= mag * Fraction(1, 2 ** 50)
    # the full product is the matrix product (library routine)
    full = oracle.gemm_sampled(Xd, Wd)
    assert np.allclose(full, Xd @ Wd.T, rtol=1e-12, atol=1e-12)


# --- storage formats ----------------------------------------------------------------

def test_formats_roundtrip():
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 16, size=(5, 64), dtype=np.uint8)
    assert np.array_equal(formats.unpack_codes(formats.pack_codes(codes)), codes)
    assert formats.pack_codes(np.array([[1, 2]], np.uint8))[0, 0] == 0x21
    for rows, nb in [(1, 1), (130, 9), (256, 128)]:
        plain = rng.integers(0, 255, size=(rows, nb), dtype=np.uint8)
        tiled = formats.tile_scales(plain)
        assert tiled.size == formats.scale_bytes(rows, nb)
        assert np.array_equal(formats.untile_scales(tiled, rows, nb), plain)
        idx = formats.scale_index(rows, nb).reshape(-1)
        assert np.unique(idx).size == idx.size
    I = formats.scale_index(256, 12)
    nbp4 = 3
    assert I[0, 0] == 0 and I[1, 0] == 16 and I[32, 0] == 4 and I[0, 1] == 1
    assert I[0, 4] == 512 and I[128, 0] == nbp4 * 512 and I[31, 3] == 31 * 16 + 3


# --- factor sizes other than 8 x 8 shared / 4 x 4 private --------------------------
# The review's size study and the note's Key Designs 2 vary the shared factor's
# size s (A is s x s, each B_b is (32/s) x (32/s)); s = 32 leaves one scalar per
# block (a shared 32 x 32 transform, scaled), s = 1 a fully private 32 x 32 block.

SIZES = (1, 2, 4, 8, 16, 32)


@pytest.mark.parametrize("s", SIZES)
def test_kron_block_all_sizes(s):
    A, B, _, _ = wl.random_factors(2, seed=20 + s, shared=s)
    t = 32 // s
    A64 = A.astype(np.float64)
    for b in range(2):
        P = oracle.kron_block(B[b], A)
        assert np.array_equal(P, np.kron(B[b].astype(np.float64), A64))
        # block (i, j) of P is B_b[i][j] times A
        i, j = t - 1, 0
        assert np.array_equal(P[s * i:s * i + s, s * j:s * j + s], B[b][i, j] * A64)


@pytest.mark.parametrize("s", SIZES)
def test_transform_factored_all_sizes(s):
    """x P_b equals the block-diagonal matmul and vec_row(B_b^T X_r A), X_r = x as t x s."""
    nb, rows = 4, 24
    A, B, _, _ = wl.random_factors(nb, seed=30 + s, shared=s)
    t = 32 // s
    X = wl.random_bf16((rows, 32 * nb), seed=31 + s, scale=3.0)
    Xd = _bf16_to_f64(X)
    Y = oracle.transform_f64(X, A, B)
    P = scipy.linalg.block_diag(*[np.kron(B[b].astype(np.float64), A.astype(np.float64))
                                  for b in range(nb)])
    ref = Xd @ P
    assert np.max(np.abs(Y - ref)) <= 1e-13 * np.max(np.abs(ref))
    for b in range(nb):
        Xr = Xd[:, 32 * b:32 * b + 32].reshape(rows, t, s)
        fac = (B[b].astype(np.float64).T[None] @ Xr @ A.astype(np.float64)[None]).reshape(rows, 32)
        assert np.max(np.abs(Y[:, 32 * b:32 * b + 32] - fac)) <= 1e-13 * np.max(np.abs(fac))
    assert np.array_equal(oracle.transform(X, A, B), Y.astype(np.float32))


@pytest.mark.parametrize("s", SIZES)
def test_inverse_fusion_all_sizes(s):
    nb = 4
    A, B, _, _ = wl.random_factors(nb, seed=40 + s, shared=s)
    X = wl.random_bf16((16, 32 * nb), seed=41 + s)
    W = wl.random_bf16((8, 32 * nb), seed=42 + s)
    got = oracle.transform_f64(X, A, B) @ oracle.weight_transform_f64(W, A, B).T
    ref = _bf16_to_f64(X) @ _bf16_to_f64(W).T
    assert np.linalg.norm(got - ref) <= 1e-10 * np.linalg.norm(ref)


def test_extreme_sizes_closed_forms():
    """s = 32: P_b = beta_b A; s = 1: P_b = alpha B_b."""
    nb = 3
    X = wl.random_bf16((8, 32 * nb), seed=50)
    Xd = _bf16_to_f64(X).reshape(8, nb, 32)
    A, B, _, _ = wl.random_factors(nb, seed=51, shared=32)
    assert B.shape == (nb, 1, 1)
    Y = oracle.transform_f64(X, A, B).reshape(8, nb, 32)
    for b in range(nb):
        ref = float(B[b, 0, 0]) * (Xd[:, b] @ A.astype(np.float64))
        assert np.allclose(Y[:, b], ref, rtol=1e-13, atol=1e-13)
    A, B, _, _ = wl.random_factors(nb, seed=52, shared=1)
    assert A.shape == (1, 1)
    Y = oracle.transform_f64(X, A, B).reshape(8, nb, 32)
    for b in range(nb):
        ref = float(A[0, 0]) * (Xd[:, b] @ B[b].astype(np.float64))
        assert np.allclose(Y[:, b], ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("s", SIZES)
def test_block_hadamard_every_size(s):
    """Normalised Sylvester Hadamards H_t/sqrt(t) (x) H_s/sqrt(s) = H_32/sqrt(32) for
    every split, so each size gives BRQ's 32-point block rotation; the weight side
    equals the activation side because that block is orthonormal and symmetric."""
    t = 32 // s
    A = (scipy.linalg.hadamard(s) / np.sqrt(s)).astype(np.float32)
    nb = 4
    B = np.repeat((scipy.linalg.hadamard(t) / np.sqrt(t))[None].astype(np.float32), nb, axis=0)
    H32 = scipy.linalg.hadamard(32) / np.sqrt(32.0)
    assert np.allclose(oracle.kron_block(B[0], A), H32, atol=1e-7)
    X = wl.random_bf16((8, 32 * nb), seed=60 + s)
    Y = oracle.transform_f64(X, A, B)
    Xd = _bf16_to_f64(X)
    assert np.allclose(Y.reshape(8, nb, 32), Xd.reshape(8, nb, 32) @ H32, atol=1e-5)
    assert np.allclose(oracle.weight_transform_f64(X, A, B), Y, rtol=1e-6, atol=1e-6)


def test_factor_shape_errors():
    A, B, _, _ = wl.random_factors(2, seed=70, shared=4)
    X = wl.random_bf16((2, 64), seed=71)
    with pytest.raises(ValueError):
        oracle.transform_f64(X, A, B[:, :2, :2])
    with pytest.raises(ValueError):
        oracle.transform_f64(X, np.eye(3, dtype=np.float32), B)
    with pytest.raises(np.linalg.LinAlgError):
        Bs = B.copy()
        Bs[1] = 0.0
        oracle.weight_transform_f64(X, A, Bs)


# --- MXFP8 (E4M3) activations: the W4A8 settings ------------------------------------
# The note (Loss & Training) names W4A8 with "MXFP8 uses E4M3"; the element format
# is OCP FP8 E4M3 (bias 7, no infinities, 448 the largest finite value).

def test_e4m3_decode_table_matches_torch():
    import torch
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    mine = oracle.e4m3_value(np.arange(256))
    fin = np.isfinite(dec)
    assert np.array_equal(np.isfinite(mine), fin)
    assert np.array_equal(mine[fin], dec[fin].astype(np.float64))
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6


def _e4m3_edges() -> np.ndarray:
    """Every midpoint between adjacent finite E4M3 magnitudes, one fp32 ulp either
    side of it, and the magnitudes themselves."""
    mags = oracle.e4m3_value(np.arange(127)).astype(np.float32)
    mids = ((mags[:-1].astype(np.float64) + mags[1:]) / 2).astype(np.float32)
    pts = np.concatenate([mags, mids, np.nextafter(mids, np.float32(np.inf)),
                          np.nextafter(mids, np.float32(0))])
    return np.concatenate([pts, -pts]).astype(np.float32)


def test_e4m3_encode_matches_torch():
    """RNE conversion against torch's float8_e4m3fn cast (a library routine) for
    |v| <= 448 plus the tie at 464; torch turns larger values into NaN, the oracle
    saturates them to 448 (checked separately)."""
    import torch
    rng = np.random.default_rng(7)
    top = int(np.float32(448.0).view(np.uint32))
    bits = rng.integers(0, top + 1, size=1 << 20, dtype=np.uint32)
    bits[: 1 << 19] |= np.uint32(0x80000000)
    v = np.concatenate([bits.view(np.float32), _e4m3_edges(), np.float32([464.0, -464.0, 0.0, -0.0])])
    got = oracle.e4m3_encode(v)
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])
    big = np.float32([464.5, 480.0, 512.0, 1e6, 3.4e38, -500.0])
    assert np.array_equal(oracle.e4m3_encode(big), np.uint8([0x7E] * 5 + [0xFE]))


def _e4m3_by_binade(v: np.ndarray) -> np.ndarray:
    """E4M3 as a 3-mantissa-bit float, written independently: below 2^-6 the step is
    2^-9, in [2^k, 2^(k+1)) it is 2^(k-3); np.rint ties to even; saturate at 448."""
    a = np.abs(v.astype(np.float64))
    with np.errstate(divide="ignore"):
        k = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    step = np.where(a < 2.0 ** -6, 2.0 ** -9, np.exp2(k - 3))
    q = np.minimum(np.rint(a / step) * step, 448.0)
    table = oracle.e4m3_value(np.arange(127))
    code = np.searchsorted(table, q).astype(np.uint8)
    assert np.all(table[code] == q)
    return code | (np.signbit(v).astype(np.uint8) << 7)


def test_e4m3_encode_by_binade():
    rng = np.random.default_rng(8)
    v = np.concatenate([(rng.standard_normal(1 << 18) * np.exp2(rng.uniform(-12, 10, 1 << 18))),
                        rng.uniform(-600, 600, 1 << 16)]).astype(np.float32)
    v = np.concatenate([v, _e4m3_edges()])
    assert np.array_equal(oracle.e4m3_encode(v), _e4m3_by_binade(v))


def test_mxfp8_scale_rule_and_rtn():
    """Identity factors and no clip: MXFP8 RTN of X by an independent numpy quantizer;
    the block maximum lands in [256, 512) times the scale (e = floor(log2 amax) - 8)."""
    inp = wl.make_inputs("tiny")
    nb = inp.B.shape[0]
    A = np.eye(8, dtype=np.float32)
    B = np.repeat(np.eye(4, dtype=np.float32)[None], nb, axis=0)
    Y, codes, scales = oracle.quantize_act(inp.X, A, B, None, None, fmt="e4m3")
    x = wl.bf16_bits_to_f32(inp.X)
    rows, K = x.shape
    blocks = x.reshape(rows, nb, 32).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    e = np.clip(np.floor(np.log2(amax)) - 8, -127, 127)
    assert np.array_equal(scales.astype(np.int64) - 127, e.astype(np.int64))
    v = (blocks / np.exp2(e)[..., None]).astype(np.float32).reshape(rows, K)
    v = np.where(v == 0, np.float32(0.0), v)
    assert np.array_equal(codes, _e4m3_by_binade(v))
    ratio = amax / np.exp2(e)
    assert np.all((ratio >= 256) & (ratio < 512))
    deq = oracle.dequantize(codes, scales, "e4m3")
    rel = np.abs(deq - x) / np.repeat(amax, 32, axis=1)
    # a half step of the top binade is at most amax / 16; a block maximum in [448, 512) x 2^e
    # saturates to 448 x 2^e, at most amax / 8 away
    assert rel.max() <= 2.0 ** -3


def test_mxfp8_linear_error_below_mxfp4():
    """W4A8 sits between W4A4 and the unquantized product (the settings' ordering)."""
    inp = wl.make_inputs("tiny")
    ref = _bf16_to_f64(inp.X) @ _bf16_to_f64(inp.W).T
    e4 = np.linalg.norm(oracle.linear(inp.X, inp.W, inp.A, inp.B, inp.g_lo, inp.g_hi) - ref)
    e8 = np.linalg.norm(oracle.linear(inp.X, inp.W, inp.A, inp.B, inp.g_lo, inp.g_hi,
                                      act_fmt="e4m3") - ref)
    assert e8 < e4


# --- KV-cache path (KV8 / KV4) ------------------------------------------------------

@pytest.mark.parametrize("s", SIZES)
def test_inverse_factors_invert_the_block(s):
    """B_b^-1 (x) A^-1 is the inverse of B_b (x) A: transforming back recovers x
    (checked against numpy's inverse of the explicit block-diagonal P)."""
    nb = 4
    A, B, _, _ = wl.random_factors(nb, seed=80 + s, shared=s)
    Ai = oracle.inverse(A.astype(np.float64))
    Bi = np.stack([oracle.inverse(B[b].astype(np.float64)) for b in range(nb)])
    Xd = wl.bf16_bits_to_f32(wl.random_bf16((6, 32 * nb), seed=81 + s)).astype(np.float64)
    Y = oracle.transform_vals_f64(Xd, A, B)
    P = scipy.linalg.block_diag(*[np.kron(B[b].astype(np.float64), A.astype(np.float64))
                                  for b in range(nb)])
    # the factors are passed as fp32; compare against the fp32-rounded inverse factors' block
    Pi = scipy.linalg.block_diag(*[np.kron(Bi[b].astype(np.float32).astype(np.float64),
                                           Ai.astype(np.float32).astype(np.float64)) for b in range(nb)])
    back = oracle.transform_vals_f64(Y, Ai.astype(np.float32), Bi.astype(np.float32))
    assert np.allclose(back, Y @ Pi, rtol=0, atol=1e-12 * np.abs(Y).max())
    assert np.allclose(np.linalg.inv(P), Pi, atol=1e-5)
    assert np.max(np.abs(back - Xd)) <= 1e-5 * np.max(np.abs(Xd))


def _mxfp8_rtn(x: np.ndarray):
    rows, K = x.shape
    blocks = x.reshape(rows, K // 32, 32).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    with np.errstate(divide="ignore"):
        e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 8, -127)
    e = np.clip(e, -127, 127)
    v = (blocks / np.exp2(e)[..., None]).astype(np.float32).reshape(rows, K)
    v = np.where(v == 0, np.float32(0.0), v)
    return _e4m3_by_binade(v), (e + 127).astype(np.uint8)


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_kv_identity_is_rtn_and_scatter(fmt):
    """Identity factors, no clip: each head vector is plain MX RTN (KV8 / KV4), stored at
    its slot; slot -1 and slots no token names keep their old contents."""
    T, H, D, S = 5, 3, 64, 9
    kv = wl.random_bf16((T, H, D), seed=90, scale=2.0)
    A = np.eye(8, dtype=np.float32)
    B = np.repeat(np.eye(4, dtype=np.float32)[None], D // 32, axis=0)
    slots = np.array([4, -1, 0, 8, 2])
    cc = np.full((S, H, D), 0x5A, np.uint8)
    cs = np.full((S, H, D // 32), 0xA5, np.uint8)
    oracle.kv_quantize(kv, A, B, None, None, fmt, slots, cc, cs)
    x = wl.bf16_bits_to_f32(kv).reshape(T * H, D)
    rc, rs = _mxfp8_rtn(x) if fmt == "e4m3" else _rtn_mxfp4(x)
    rc, rs = rc.reshape(T, H, D), rs.reshape(T, H, D // 32)
    for t, sl in enumerate(slots):
        if sl >= 0:
            assert np.array_equal(cc[sl], rc[t]) and np.array_equal(cs[sl], rs[t])
    for sl in (1, 3, 5, 6, 7):
        assert np.all(cc[sl] == 0x5A) and np.all(cs[sl] == 0xA5)


def test_kv_head_locality():
    """Changing one head of one token changes only that head's cache entry."""
    T, H, D = 4, 4, 128
    kv = wl.random_bf16((T, H, D), seed=91)
    A, B, g_lo, g_hi = wl.random_factors(D // 32, seed=92)
    slots = np.arange(T)
    c0 = np.zeros((T, H, D), np.uint8); s0 = np.zeros((T, H, D // 32), np.uint8)
    c1 = c0.copy(); s1 = s0.copy()
    oracle.kv_quantize(kv, A, B, g_lo, g_hi, "e4m3", slots, c0, s0)
    kv2 = kv.copy()
    kv2[2, 1] = wl.random_bf16((D,), seed=93, scale=10.0)
    oracle.kv_quantize(kv2, A, B, g_lo, g_hi, "e4m3", slots, c1, s1)
    diff = np.any(c0 != c1, axis=2) | np.any(s0 != s1, axis=2)
    assert diff[2, 1] and diff.sum() == 1


def test_kv_roundtrip_with_inverse_factors():
    """Dequantizing the cache through B^-1 (x) A^-1 gives back K within the MX error;
    the transposed inverse (a plausible orientation slip) does not."""
    T, H, D = 16, 2, 128
    kv = wl.random_bf16((T, H, D), seed=94, scale=1.5)
    A, B, _, _ = wl.random_factors(D // 32, seed=95)
    Ai = oracle.inverse(A.astype(np.float64)).astype(np.float32)
    Bi = np.stack([oracle.inverse(b.astype(np.float64)) for b in B]).astype(np.float32)
    x = wl.bf16_bits_to_f32(kv).astype(np.float64)
    for fmt, tol in (("e4m3", 0.05), ("e2m1", 0.25)):
        cc = np.zeros((T, H, D), np.uint8); cs = np.zeros((T, H, D // 32), np.uint8)
        oracle.kv_quantize(kv, A, B, None, None, fmt, np.arange(T), cc, cs)
        back = oracle.kv_dequantize(cc, cs, np.arange(T), fmt, Ai, Bi)
        rel = np.linalg.norm(back - x) / np.linalg.norm(x)
        assert rel < tol, (fmt, rel)
        wrong = oracle.kv_dequantize(cc, cs, np.arange(T), fmt, Ai.T.copy(),
                                     np.ascontiguousarray(Bi.transpose(0, 2, 1)))
        assert np.linalg.norm(wrong - x) / np.linalg.norm(x) > 2 * rel

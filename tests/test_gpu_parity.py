"""CUDA path vs the CPU oracle, element by element, through the C-ABI.

Bars (BATQuant W4A4 linear; readings of the pages as stated in the oracle):
  * E2M1 codes and UE8M0 scale bytes: bit-exact when the oracle quantizer is fed
    the GPU's fp32 transformed values and the GPU's fp32 clip ratios;
  * transformed values: block-normwise |y_gpu - y_ref|_inf <= 1e-5 |y_ref|_inf;
  * GEMM: relative Frobenius error <= 1e-3 against the oracle's fp64 product of
    the same dequantized operands (fp32 output), and bf16 output against the
    bf16-rounded fp64 product.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import formats
import workloads as wl

pytestmark = pytest.mark.gpu

TRANSFORM_TOL = 1e-5
GEMM_TOL = 1e-3


@pytest.fixture(scope="module")
def bat():
    import w4a4_bit_gemm_b200 as m
    m.lib()
    return m


def _dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def _dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def _host(q, rows, K):
    codes = formats.unpack_codes(q.codes.cpu().numpy().reshape(rows, K // 2))
    tiled = q.scales.cpu().numpy()
    scales = formats.untile_scales(tiled, rows, K // 32)
    return codes, scales, tiled


def _check_transform(y_gpu: np.ndarray, y_ref: np.ndarray):
    rows, K = y_ref.shape
    g = y_gpu.reshape(rows, K // 32, 32).astype(np.float64)
    r = y_ref.reshape(rows, K // 32, 32).astype(np.float64)
    err = np.max(np.abs(g - r), axis=2)
    ref = np.max(np.abs(r), axis=2)
    bad = err > TRANSFORM_TOL * ref
    assert not bad.any(), (np.argwhere(bad)[:5], (err / np.maximum(ref, 1e-300)).max())


def _run_act(bat, X, A, B, g_lo, g_hi):
    Xd = _dev_bf16(X)
    Ad, Bd = _dev_f32(A), _dev_f32(B)
    gl = None if g_lo is None else _dev_f32(g_lo)
    gh = None if g_hi is None else _dev_f32(g_hi)
    Xq, y = bat.bat_quantize_act_trace(Xd, Ad, Bd, gl, gh)
    Xq2 = bat.bat_quantize_act(Xd, Ad, Bd, gl, gh)
    torch.cuda.synchronize()
    assert torch.equal(Xq.codes, Xq2.codes) and torch.equal(Xq.scales, Xq2.scales)
    nb = X.shape[1] // 32
    r_lo = bat.bat_clip_ratios(gl, nb).cpu().numpy()
    r_hi = bat.bat_clip_ratios(gh, nb).cpu().numpy()
    return Xq, y.cpu().numpy(), r_lo, r_hi


def _check_act(bat, X, A, B, g_lo, g_hi):
    rows, K = X.shape
    Xq, y_gpu, r_lo, r_hi = _run_act(bat, X, A, B, g_lo, g_hi)
    nb = K // 32
    assert np.array_equal(r_lo, oracle.clip_ratios(g_lo, nb))
    assert np.array_equal(r_hi, oracle.clip_ratios(g_hi, nb))
    _check_transform(y_gpu, oracle.transform(X, A, B))
    codes, scales, tiled = _host(Xq, rows, K)
    oc, os_, bad = oracle.quantize(y_gpu, r_lo, r_hi)
    assert bad == 0
    mism = np.argwhere(codes != oc)
    assert mism.size == 0, (mism[:5], codes[tuple(mism[0])], oc[tuple(mism[0])])
    assert np.array_equal(scales, os_)
    assert np.all(tiled[formats.padding_mask(rows, nb)] == 0)
    return Xq, codes, scales


# ---------------------------------------------------------------- element conversion
def test_e2m1_conversion_every_fp32_up_to_8(bat):
    top = int(np.float32(8.0).view(np.uint32))
    step = 1 << 26
    for start in range(0, top + 1, step):
        bits = np.arange(start, min(start + step, top + 1), dtype=np.uint32)
        v = bits.view(np.float32)
        got = bat.bat_e2m1_encode(_dev_f32(v)).cpu().numpy()
        assert np.array_equal(got, oracle.e2m1_encode(v)), start
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 0x7F800000, size=1 << 22, dtype=np.uint32) | np.uint32(0x80000000)
    v = np.concatenate([bits.view(np.float32), np.array([-0.0, 0.0, -1e-30, 1e-30, -7.0, 1e30], np.float32)])
    got = bat.bat_e2m1_encode(_dev_f32(v)).cpu().numpy()
    assert np.array_equal(got, oracle.e2m1_encode(v))


def test_clip_ratios(bat):
    g = np.concatenate([np.linspace(-20, 20, 4001, dtype=np.float32),
                        np.array([np.inf, 0.0, 1e-8], np.float32)])
    r = bat.bat_clip_ratios(_dev_f32(g)).cpu().numpy()
    assert np.array_equal(r, oracle.clip_ratios(g))
    assert np.all(bat.bat_clip_ratios(None, 7).cpu().numpy() == 1.0)


# ---------------------------------------------------------------- prologue
@pytest.mark.parametrize("name", wl.ORDER)
def test_quantize_act_workloads(bat, name):
    inp = wl.make_inputs(name, with_weight=False)
    _check_act(bat, inp.X, inp.A, inp.B, inp.g_lo, inp.g_hi)


@pytest.mark.parametrize("M,K", [(1, 32), (1, 4096), (17, 96), (130, 160), (3, 1056), (129, 4128),
                                 (64, 1024 + 96), (65, 4128), (16, 12288), (2, 262144)])
def test_quantize_act_ragged(bat, M, K):
    X = wl.random_bf16((M, K), seed=M * 7 + K, scale=3.0)
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=K)
    _check_act(bat, X, A, B, g_lo, g_hi)


def test_quantize_act_no_clip_identity_is_rtn(bat):
    """Identity factors and no clip give plain MXFP4 round-to-nearest of X."""
    inp = wl.make_inputs("tiny", with_weight=False)
    nb = inp.B.shape[0]
    A = np.eye(8, dtype=np.float32)
    B = np.repeat(np.eye(4, dtype=np.float32)[None], nb, axis=0)
    Xq, codes, scales = _check_act(bat, inp.X, A, B, None, None)
    _, oc, os_ = oracle.quantize_act(inp.X, A, B, None, None)
    assert np.array_equal(codes, oc) and np.array_equal(scales, os_)


def test_quantize_act_zero_and_constant_rows(bat):
    M, K = 8, 256
    X = np.zeros((M, K), np.uint16)
    X[1] = wl.f32_to_bf16_bits(np.full(K, -2.5, np.float32))
    X[2, :32] = wl.f32_to_bf16_bits(np.full(32, 1e-30, np.float32))
    X[3] = wl.f32_to_bf16_bits(np.full(K, 1e30, np.float32))
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=4)
    _check_act(bat, X, A, B, g_lo, g_hi)


# ---------------------------------------------------------------- weight side
@pytest.mark.parametrize("clip", [False, True])
@pytest.mark.parametrize("N,K", [(128, 256), (200, 96), (1, 4096), (384, 4096)])
def test_prepare_weight(bat, N, K, clip):
    W = wl.random_bf16((N, K), seed=N + K, scale=0.02)
    A, B, _, _ = wl.random_factors(K // 32, seed=K + 1)
    rng = np.random.default_rng(N)
    gw_lo = rng.uniform(1, 4, size=(N, K // 32)).astype(np.float32) if clip else None
    gw_hi = rng.uniform(1, 4, size=(N, K // 32)).astype(np.float32) if clip else None
    wt = torch.empty(N, K, dtype=torch.float32, device="cuda")
    Wq = bat.bat_prepare_weight(_dev_bf16(W), _dev_f32(A), _dev_f32(B),
                                None if gw_lo is None else _dev_f32(gw_lo),
                                None if gw_hi is None else _dev_f32(gw_hi), wt_out=wt)
    torch.cuda.synchronize()
    wt_gpu = wt.cpu().numpy()
    _check_transform(wt_gpu, oracle.weight_transform_f64(W, A, B).astype(np.float32))
    r_lo = None if gw_lo is None else oracle.clip_ratios(gw_lo.reshape(-1)).reshape(N, -1)
    r_hi = None if gw_hi is None else oracle.clip_ratios(gw_hi.reshape(-1)).reshape(N, -1)
    oc, os_, _ = oracle.quantize(wt_gpu, r_lo, r_hi, per_row=True)
    codes, scales, tiled = _host(Wq, N, K)
    assert np.array_equal(codes, oc)
    assert np.array_equal(scales, os_)
    assert np.all(tiled[formats.padding_mask(N, K // 32)] == 0)


def test_prepare_weight_singular(bat):
    K = 64
    W = wl.random_bf16((8, K), seed=1)
    A, B, _, _ = wl.random_factors(K // 32, seed=2)
    B[1] = 0.0
    with pytest.raises(bat.BatError) as e:
        bat.bat_prepare_weight(_dev_bf16(W), _dev_f32(A), _dev_f32(B))
    assert e.value.status == 4



# ---------------------------------------------------------------- other factor splits
SHARED_SIZES = (1, 2, 4, 8, 16, 32)


def _check_act_gpk(bat, X, A, B, g_lo, g_hi):
    rows, K = X.shape
    nb = K // 32
    Xd, Ad, Bd = _dev_bf16(X), _dev_f32(A), _dev_f32(B)
    gl = None if g_lo is None else _dev_f32(g_lo)
    gh = None if g_hi is None else _dev_f32(g_hi)
    y = torch.empty(rows, K, dtype=torch.float32, device="cuda")
    Xq = bat.bat_quantize_act_gpk(Xd, Ad, Bd, gl, gh, y_out=y)
    Xq2 = bat.bat_quantize_act_gpk(Xd, Ad, Bd, gl, gh)
    torch.cuda.synchronize()
    assert torch.equal(Xq.codes, Xq2.codes) and torch.equal(Xq.scales, Xq2.scales)
    y_gpu = y.cpu().numpy()
    _check_transform(y_gpu, oracle.transform(X, A, B))
    r_lo = bat.bat_clip_ratios(gl, nb).cpu().numpy()
    r_hi = bat.bat_clip_ratios(gh, nb).cpu().numpy()
    oc, os_, bad = oracle.quantize(y_gpu, r_lo, r_hi)
    assert bad == 0
    codes, scales, tiled = _host(Xq, rows, K)
    assert np.array_equal(codes, oc)
    assert np.array_equal(scales, os_)
    assert np.all(tiled[formats.padding_mask(rows, nb)] == 0)
    return Xq, y_gpu


@pytest.mark.parametrize("s", SHARED_SIZES)
@pytest.mark.parametrize("M,K", [(130, 1056), (3, 4128), (257, 256)])
def test_quantize_act_gpk_sizes(bat, s, M, K):
    X = wl.random_bf16((M, K), seed=M + K + s, scale=3.0)
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=K + s, shared=s)
    _check_act_gpk(bat, X, A, B, g_lo, g_hi)


def test_quantize_act_gpk_default_split_matches(bat):
    """s = 8 through the generic entry point is bat_quantize_act, bit for bit."""
    inp = wl.make_inputs("tiny", with_weight=False)
    Xd, Ad, Bd = _dev_bf16(inp.X), _dev_f32(inp.A), _dev_f32(inp.B)
    gl, gh = _dev_f32(inp.g_lo), _dev_f32(inp.g_hi)
    q1 = bat.bat_quantize_act(Xd, Ad, Bd, gl, gh)
    q2 = bat.bat_quantize_act_gpk(Xd, Ad, Bd, gl, gh)
    torch.cuda.synchronize()
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.scales, q2.scales)


@pytest.mark.parametrize("s", SHARED_SIZES)
def test_prepare_weight_gpk_sizes(bat, s):
    N, K = 136, 1056
    W = wl.random_bf16((N, K), seed=N + K + s, scale=0.02)
    A, B, _, _ = wl.random_factors(K // 32, seed=K + 1 + s, shared=s)
    rng = np.random.default_rng(s)
    gw_lo = rng.uniform(1, 4, size=(N, K // 32)).astype(np.float32)
    gw_hi = rng.uniform(1, 4, size=(N, K // 32)).astype(np.float32)
    wt = torch.empty(N, K, dtype=torch.float32, device="cuda")
    Wq = bat.bat_prepare_weight_gpk(_dev_bf16(W), _dev_f32(A), _dev_f32(B), _dev_f32(gw_lo),
                                    _dev_f32(gw_hi), wt_out=wt)
    torch.cuda.synchronize()
    wt_gpu = wt.cpu().numpy()
    _check_transform(wt_gpu, oracle.weight_transform_f64(W, A, B).astype(np.float32))
    r_lo = oracle.clip_ratios(gw_lo.reshape(-1)).reshape(N, -1)
    r_hi = oracle.clip_ratios(gw_hi.reshape(-1)).reshape(N, -1)
    oc, os_, _ = oracle.quantize(wt_gpu, r_lo, r_hi, per_row=True)
    codes, scales, tiled = _host(Wq, N, K)
    assert np.array_equal(codes, oc)
    assert np.array_equal(scales, os_)


def test_gpk_errors(bat):
    X = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    A = torch.eye(3, device="cuda")
    B = torch.eye(4, device="cuda").repeat(2, 1, 1).contiguous()
    Xq = bat.MXFP4.empty(4, 64)
    st = bat.lib().bat_quantize_act_gpk(bat._ptr(X), 4, 64, bat._ptr(A), 3, bat._ptr(B), None, None,
                                        bat.ctypes.byref(Xq.struct()), None, bat._stream(None))
    assert st == 6  # BAT_ERR_UNSUPPORTED
    A, B, _, _ = wl.random_factors(2, seed=3, shared=2)
    B[1] = 0.0
    with pytest.raises(bat.BatError) as e:
        bat.bat_prepare_weight_gpk(_dev_bf16(wl.random_bf16((8, 64), seed=4)), _dev_f32(A), _dev_f32(B))
    assert e.value.status == 4
    assert bat.bat_device_error() == 0


def test_block_hadamard_mode(bat):
    """Every split of the normalised Sylvester Hadamard gives the same 32-point block
    rotation (the BRQ article's block rotation), in fp32 to the bit: the factor
    products are powers of two times fp32(1/sqrt 2) or exact. Checked against the
    oracle, and the whole linear layer against the oracle's fp64 product."""
    M, N, K = 200, 264, 1056
    X = wl.random_bf16((M, K), seed=5, scale=3.0)
    W = wl.random_bf16((N, K), seed=6, scale=0.02)
    nb = K // 32
    outs = []
    for s in SHARED_SIZES:
        A, B = bat.bat_block_hadamard_factors(s, nb)
        Xq, y = _check_act_gpk(bat, X, A.numpy(), B.numpy(), None, None)
        outs.append((Xq, y))
    for Xq, y in outs[1:]:
        assert torch.equal(Xq.codes, outs[0][0].codes) and torch.equal(Xq.scales, outs[0][0].scales)
        assert np.array_equal(y, outs[0][1])
    A, B = bat.bat_block_hadamard_factors(4, nb)
    Wq = bat.bat_prepare_weight_gpk(_dev_bf16(W), A.cuda(), B.cuda())
    Y = bat.bat_mxfp4_gemm(outs[2][0], Wq, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.linear(X, W, A.numpy(), B.numpy(), None, None)
    rel = np.linalg.norm(Y.cpu().numpy() - ref) / np.linalg.norm(ref)
    assert rel <= 1e-2, rel  # codes may differ where the two transforms round to a tie
    # and exactly, on the GPU's own codes
    _gemm_check(bat, outs[2][0], Wq, M, N, K)

# ---------------------------------------------------------------- GEMM
def _check_outputs(y32, y16, Xd, Wd):
    """Sampled outputs against the oracle's fp64 product of the same dequantized
    operands (Xd, Wd: the sampled rows and columns): relative Frobenius error, a
    per-element bound far inside fp32 accumulation of the absolute terms, and the
    bf16 output against the bf16-rounded product."""
    ref = oracle.gemm_sampled(Xd, Wd)
    assert np.all(np.isfinite(y32))
    rel = np.linalg.norm(y32 - ref) / max(np.linalg.norm(ref), 1e-300)
    assert rel <= GEMM_TOL, rel
    mag = oracle.gemm_sampled(np.abs(Xd), np.abs(Wd))
    assert np.all(np.abs(y32 - ref) <= 1e-5 * mag + 1e-30), np.max(np.abs(y32 - ref) / (mag + 1e-30))
    if y16 is not None:
        ref16 = torch.from_numpy(ref).to(torch.bfloat16).float().numpy().astype(np.float64)
        rel16 = np.linalg.norm(y16 - ref16) / max(np.linalg.norm(ref16), 1e-300)
        assert rel16 <= GEMM_TOL, rel16
    return rel


def _gemm_check(bat, Xq, Wq, M, N, K, rows=None, cols=None):
    xc, xs, _ = _host(Xq, M, K)
    wc, ws, _ = _host(Wq, N, K)
    r = np.arange(M) if rows is None else np.asarray(rows)
    c = np.arange(N) if cols is None else np.asarray(cols)
    Xd = oracle.dequantize(xc[r], xs[r])
    Wd = oracle.dequantize(wc[c], ws[c])
    Y32 = bat.bat_mxfp4_gemm(Xq, Wq, out_dtype=torch.float32)
    Y16 = bat.bat_mxfp4_gemm(Xq, Wq, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    y32 = Y32.cpu().numpy()[np.ix_(r, c)].astype(np.float64)
    y16 = Y16.float().cpu().numpy()[np.ix_(r, c)].astype(np.float64)
    return _check_outputs(y32, y16, Xd, Wd)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (64, 128, 256), (1, 8, 32), (17, 200, 96),
                                   (130, 300, 160), (256, 512, 1024), (200, 264, 4128),
                                   (300, 1000, 2048),
                                   # one row of tiles: split-K over a cluster per tile
                                   (1, 256, 2048), (100, 520, 1024), (128, 1000, 768),
                                   (33, 300, 2080), (16, 6144, 4096),
                                   # decode kernel: eight K stages per CTA, 48 token rows
                                   (5, 136, 16384), (48, 1000, 4128),
                                   # CTA pairs: 256 x 256 tiles, ragged rows, columns and K
                                   (512, 768, 2048), (384, 256, 1056), (129, 136, 32),
                                   (1000, 1288, 4128)])
def test_gemm_shapes(bat, M, N, K):
    X = wl.random_bf16((M, K), seed=M + 3 * K, scale=2.0)
    W = wl.random_bf16((N, K), seed=N + 5 * K, scale=0.02)
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=K + 9)
    Xq = bat.bat_quantize_act(_dev_bf16(X), _dev_f32(A), _dev_f32(B), _dev_f32(g_lo), _dev_f32(g_hi))
    Wq = bat.bat_prepare_weight(_dev_bf16(W), _dev_f32(A), _dev_f32(B))
    _gemm_check(bat, Xq, Wq, M, N, K)


def _sample(n, count, seed, tile=None):
    """Edge indices, `count` random ones and, with `tile`, one random index inside
    every tile of that size (so every output tile of the GEMM is checked)."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, n // 2, n - 1] + ([127, 128] if n > 128 else [])
    parts = [fixed, rng.integers(0, n, size=count)]
    if tile:
        starts = np.arange(0, n, tile)
        parts.append(starts + rng.integers(0, tile, size=starts.size) % (n - starts))
        parts.append(np.minimum(starts + tile - 1, n - 1))  # last row/column of each tile
    return np.unique(np.concatenate(parts)).astype(np.int64)


@pytest.mark.parametrize("name", wl.ORDER)
def test_linear_workloads(bat, name):
    """bat_linear at the full workload sizes, as the benchmark launches it; sampled outputs."""
    inp = wl.make_inputs(name)
    w = wl.WORKLOADS[name]
    Xd = _dev_bf16(inp.X)
    Ad, Bd = _dev_f32(inp.A), _dev_f32(inp.B)
    gl, gh = _dev_f32(inp.g_lo), _dev_f32(inp.g_hi)
    Wq = bat.bat_prepare_weight(_dev_bf16(inp.W), Ad, Bd)
    Y = bat.bat_linear(Xd, Wq, Ad, Bd, gl, gh, out_dtype=torch.float32)
    Xq = bat.bat_quantize_act(Xd, Ad, Bd, gl, gh)
    Y2 = bat.bat_mxfp4_gemm(Xq, Wq, out_dtype=torch.float32)
    Y3 = bat.bat_linear(Xd, Wq, Ad, Bd, gl, gh, out_dtype=torch.float32, fused=True)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)  # unfused linear == quantize then GEMM, bit for bit
    assert torch.equal(Y, Y3)  # the tile-level overlap changes only the synchronisation
    # a row in every 128-row tile and a column in every 256-column tile, plus edges
    r = np.arange(w.M) if w.M <= 64 else _sample(w.M, 24, 1, tile=128)
    c = np.arange(w.N) if w.N <= 512 else _sample(w.N, 200, 2, tile=256)
    x_codes, x_scales, _ = _host(Xq, w.M, w.K)
    w_codes, w_scales, _ = _host(Wq, w.N, w.K)
    y = Y.cpu().numpy()[np.ix_(r, c)].astype(np.float64)
    _check_outputs(y, None, oracle.dequantize(x_codes[r], x_scales[r]),
                   oracle.dequantize(w_codes[c], w_scales[c]))
    # and against the oracle's own quantization of its own transform (same codes almost everywhere)
    if w.M * w.K <= 2048 * 4096:
        _, oc, os_ = oracle.quantize_act(inp.X, inp.A, inp.B, inp.g_lo, inp.g_hi)
        agree = np.mean(oc == x_codes)
        assert agree > 0.999, agree
    assert bat.bat_device_error() == 0


@pytest.mark.parametrize("M,N,K", [(300, 1000, 2048), (129, 264, 4128), (1000, 1288, 4128),
                                   (256, 512, 256), (2048, 768, 12288), (777, 520, 96)])
def test_linear_fused_equals_unfused(bat, M, N, K):
    """fused=True (the GEMM starts on each token tile as the prologue publishes it) gives
    the same codes and the same Y bytes as fused=False; one workspace reused across calls
    and shapes (stale flags of earlier calls must not release a later one)."""
    X = wl.random_bf16((M, K), seed=M + K, scale=2.0)
    W = wl.random_bf16((N, K), seed=N + 3 * K, scale=0.02)
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=K + 5)
    Xd, Ad, Bd, gl, gh = _dev_bf16(X), _dev_f32(A), _dev_f32(B), _dev_f32(g_lo), _dev_f32(g_hi)
    Wq = bat.bat_prepare_weight(_dev_bf16(W), Ad, Bd)
    ws = torch.empty(bat.bat_linear_workspace_bytes(M, K) + 4096, dtype=torch.uint8, device="cuda")
    for dt in (torch.bfloat16, torch.float32):
        ref = bat.bat_linear(Xd, Wq, Ad, Bd, gl, gh, out_dtype=dt, workspace=ws)
        codes_ref = ws.clone()
        for _ in range(3):
            got = bat.bat_linear(Xd, Wq, Ad, Bd, gl, gh, out_dtype=dt, workspace=ws, fused=True)
            torch.cuda.synchronize()
            assert torch.equal(got, ref)
        n_q = bat.bat_mxfp4_codes_bytes(M, K)
        assert torch.equal(ws[:n_q], codes_ref[:n_q])  # the same codes
    assert bat.bat_device_error() == 0


def test_argument_errors_launch_nothing(bat):
    X = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    A = torch.eye(8, device="cuda")
    B = torch.eye(4, device="cuda").repeat(2, 1, 1).contiguous()
    # a 5-row output for 4 rows of X: buffers large enough, so the library's shape check
    # (not the binding's size check) is what refuses it
    bad = bat.MXFP4.empty(5, 64)
    with pytest.raises(bat.BatError) as e:
        bat.bat_quantize_act(X, A, B, Xq=bad)
    assert e.value.status == 2
    # buffers too small for the shape they claim: refused by the binding before any call
    small = bat.MXFP4.empty(4, 64)
    with pytest.raises(ValueError):
        bat.bat_quantize_act(torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda"), A, B,
                             Xq=bat.MXFP4(small.codes, small.scales, 8, 64))
    st = bat.lib().bat_quantize_act(None, 4, 64, None, None, None, None, None, None)
    assert st == 1
    assert bat.bat_device_error() == 0


# ---------------------------------------------------------------- W4A8 (MXFP8 activations)
def _host8(q, rows, K):
    codes = q.codes.cpu().numpy().reshape(rows, K)
    tiled = q.scales.cpu().numpy()
    return codes, formats.untile_scales(tiled, rows, K // 32), tiled


def test_e4m3_conversion(bat):
    rng = np.random.default_rng(4)
    top = int(np.float32(1024.0).view(np.uint32))
    bits = rng.integers(0, top, size=1 << 22, dtype=np.uint32)
    bits[::2] |= np.uint32(0x80000000)
    mags = oracle.e4m3_value(np.arange(127)).astype(np.float32)
    mids = ((mags[:-1].astype(np.float64) + mags[1:]) / 2).astype(np.float32)
    edges = np.concatenate([mags, mids, np.nextafter(mids, np.float32(np.inf)),
                            np.nextafter(mids, np.float32(0)), np.float32([464, 465, 1e30, 0.0, -0.0])])
    v = np.concatenate([bits.view(np.float32), edges, -edges])
    got = bat.bat_e4m3_encode(_dev_f32(v)).cpu().numpy()
    assert np.array_equal(got, oracle.e4m3_encode(v))


def _check_act8(bat, X, A, B, g_lo, g_hi):
    rows, K = X.shape
    nb = K // 32
    Xd, Ad, Bd = _dev_bf16(X), _dev_f32(A), _dev_f32(B)
    gl = None if g_lo is None else _dev_f32(g_lo)
    gh = None if g_hi is None else _dev_f32(g_hi)
    y = torch.empty(rows, K, dtype=torch.float32, device="cuda")
    Xq = bat.bat_quantize_act_mxfp8(Xd, Ad, Bd, gl, gh, y_out=y)
    Xq2 = bat.bat_quantize_act_mxfp8(Xd, Ad, Bd, gl, gh)
    torch.cuda.synchronize()
    assert torch.equal(Xq.codes, Xq2.codes) and torch.equal(Xq.scales, Xq2.scales)
    y_gpu = y.cpu().numpy()
    _check_transform(y_gpu, oracle.transform(X, A, B))
    r_lo = bat.bat_clip_ratios(gl, nb).cpu().numpy()
    r_hi = bat.bat_clip_ratios(gh, nb).cpu().numpy()
    oc, os_, bad = oracle.quantize(y_gpu, r_lo, r_hi, fmt="e4m3")
    assert bad == 0
    codes, scales, tiled = _host8(Xq, rows, K)
    mism = np.argwhere(codes != oc)
    assert mism.size == 0, (mism[:5], codes[tuple(mism[0])], oc[tuple(mism[0])])
    assert np.array_equal(scales, os_)
    assert np.all(tiled[formats.padding_mask(rows, nb)] == 0)
    return Xq


@pytest.mark.parametrize("M,K", [(1, 32), (17, 96), (130, 1056), (3, 4128), (257, 256)])
def test_quantize_act_mxfp8_ragged(bat, M, K):
    X = wl.random_bf16((M, K), seed=M + 11 * K, scale=3.0)
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=K + 5)
    _check_act8(bat, X, A, B, g_lo, g_hi)


@pytest.mark.parametrize("s", [2, 4, 16])
def test_quantize_act_mxfp8_splits(bat, s):
    X = wl.random_bf16((130, 1056), seed=s, scale=3.0)
    A, B, g_lo, g_hi = wl.random_factors(1056 // 32, seed=s + 3, shared=s)
    _check_act8(bat, X, A, B, g_lo, g_hi)


@pytest.mark.parametrize("name", ["tiny", "mlp_gate_up", "mlp_down"])
def test_quantize_act_mxfp8_workloads(bat, name):
    inp = wl.make_inputs(name, with_weight=False)
    _check_act8(bat, inp.X, inp.A, inp.B, inp.g_lo, inp.g_hi)


def _w4a8_check(bat, Xq, Wq, M, N, K, rows=None, cols=None):
    xc, xs, _ = _host8(Xq, M, K)
    wc, ws, _ = _host(Wq, N, K)
    r = np.arange(M) if rows is None else np.asarray(rows)
    c = np.arange(N) if cols is None else np.asarray(cols)
    Xd = oracle.dequantize(xc[r], xs[r], "e4m3")
    Wd = oracle.dequantize(wc[c], ws[c])
    Y32 = bat.bat_w4a8_gemm(Xq, Wq, out_dtype=torch.float32)
    Y16 = bat.bat_w4a8_gemm(Xq, Wq, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    y32 = Y32.cpu().numpy()[np.ix_(r, c)].astype(np.float64)
    y16 = Y16.float().cpu().numpy()[np.ix_(r, c)].astype(np.float64)
    return _check_outputs(y32, y16, Xd, Wd)


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (1, 8, 128), (17, 200, 256), (130, 300, 512),
                                   (256, 512, 1024), (200, 264, 4096), (300, 1000, 2048),
                                   (16, 2048, 1024), (3, 300, 768)])
def test_w4a8_gemm_shapes(bat, M, N, K):
    X = wl.random_bf16((M, K), seed=M + 7 * K, scale=2.0)
    W = wl.random_bf16((N, K), seed=N + 9 * K, scale=0.02)
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=K + 2)
    Ad, Bd = _dev_f32(A), _dev_f32(B)
    Xq = bat.bat_quantize_act_mxfp8(_dev_bf16(X), Ad, Bd, _dev_f32(g_lo), _dev_f32(g_hi))
    Wq = bat.bat_prepare_weight(_dev_bf16(W), Ad, Bd)
    _w4a8_check(bat, Xq, Wq, M, N, K)
    assert bat.bat_device_error() == 0


@pytest.mark.parametrize("name", ["mlp_gate_up", "mlp_down", "prefill_o", "decode_qkv"])
def test_w4a8_linear_workloads(bat, name):
    """W4A8 at the full workload sizes: sampled outputs against the oracle, and the
    error of the layer against the unquantized product below W4A4's."""
    inp = wl.make_inputs(name)
    w = wl.WORKLOADS[name]
    Ad, Bd = _dev_f32(inp.A), _dev_f32(inp.B)
    gl, gh = _dev_f32(inp.g_lo), _dev_f32(inp.g_hi)
    Xd = _dev_bf16(inp.X)
    Wq = bat.bat_prepare_weight(_dev_bf16(inp.W), Ad, Bd)
    Xq8 = bat.bat_quantize_act_mxfp8(Xd, Ad, Bd, gl, gh)
    rows = None if w.M <= 64 else _sample(w.M, 24, 3, tile=128)
    cols = None if w.N <= 512 else _sample(w.N, 200, 4, tile=256)
    _w4a8_check(bat, Xq8, Wq, w.M, w.N, w.K, rows, cols)
    Xq4 = bat.bat_quantize_act(Xd, Ad, Bd, gl, gh)
    Y4 = bat.bat_mxfp4_gemm(Xq4, Wq, out_dtype=torch.float32)
    Y8 = bat.bat_w4a8_gemm(Xq8, Wq, out_dtype=torch.float32)
    torch.cuda.synchronize()
    r = np.arange(w.M) if rows is None else rows
    c = np.arange(w.N) if cols is None else cols
    exact = oracle.gemm_sampled(wl.bf16_bits_to_f32(inp.X).astype(np.float64),
                                wl.bf16_bits_to_f32(inp.W).astype(np.float64), r, c)
    e4 = np.linalg.norm(Y4.cpu().numpy()[np.ix_(r, c)] - exact)
    e8 = np.linalg.norm(Y8.cpu().numpy()[np.ix_(r, c)] - exact)
    assert e8 < e4, (e8, e4)
    assert bat.bat_device_error() == 0


def test_w4a8_errors(bat):
    X = torch.zeros(4, 96, dtype=torch.bfloat16, device="cuda")
    A = torch.eye(8, device="cuda")
    B = torch.eye(4, device="cuda").repeat(3, 1, 1).contiguous()
    Xq = bat.bat_quantize_act_mxfp8(X, A, B)
    Wq = bat.MXFP4.empty(8, 96)
    with pytest.raises(bat.BatError) as e:
        bat.bat_w4a8_gemm(Xq, Wq)  # K % 128 != 0
    assert e.value.status == 2
    assert bat.bat_device_error() == 0


# ---------------------------------------------------------------- KV-cache path
def _kv_host(cache, fmt):
    S, H, D = cache.num_slots, cache.H, cache.D
    raw = cache.codes.cpu().numpy()
    codes = raw.reshape(S, H, D) if fmt == "mxfp8" else \
        formats.unpack_codes(raw.reshape(S * H, D // 2)).reshape(S, H, D)
    return codes, cache.scales.cpu().numpy().reshape(S, H, D // 32)


def _kv_case(bat, T, H, D, S, fmt, s=8, clip=True, seed=0):
    kv = wl.random_bf16((T, H, D), seed=seed + 100, scale=2.0)
    A, B, g_lo, g_hi = wl.random_factors(D // 32, seed=seed + 101, shared=s)
    if not clip:
        g_lo = g_hi = None
    rng = np.random.default_rng(seed)
    slots = rng.permutation(S)[:T].astype(np.int64)
    slots[rng.random(T) < 0.2] = -1
    cache = bat.KVCache.empty(S, H, D, fmt)
    cache.codes.fill_(0x5A)
    cache.scales.fill_(0xA5)
    y = torch.empty(T, H, D, dtype=torch.float32, device="cuda")
    Ad, Bd = _dev_f32(A), _dev_f32(B)
    gl = None if g_lo is None else _dev_f32(g_lo)
    gh = None if g_hi is None else _dev_f32(g_hi)
    sd = torch.from_numpy(slots).cuda()
    bat.bat_kv_quantize(_dev_bf16(kv), Ad, Bd, sd, cache, gl, gh, y_out=y)
    torch.cuda.synchronize()
    return kv, A, B, g_lo, g_hi, slots, cache, y.cpu().numpy(), sd


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
@pytest.mark.parametrize("T,H,D,S,s", [(1, 8, 128, 4, 8), (37, 8, 128, 64, 8), (5, 3, 64, 9, 4),
                                       (4, 2, 96, 7, 2), (3, 2, 256, 5, 16), (16, 4, 128, 20, 1),
                                       (6, 2, 128, 8, 32), (511, 8, 128, 600, 8),
                                       # from 4096 (token, head) rows: the tensor-core prologue
                                       (512, 8, 128, 600, 8), (2048, 2, 96, 2100, 4),
                                       (4100, 1, 256, 4200, 16), (700, 8, 64, 800, 1)])
def test_kv_quantize_parity(bat, fmt, T, H, D, S, s):
    kv, A, B, g_lo, g_hi, slots, cache, y_gpu, _ = _kv_case(bat, T, H, D, S, fmt, s, seed=T + D)
    nb = D // 32
    _check_transform(y_gpu.reshape(T * H, D), oracle.transform(kv.reshape(T * H, D), A, B))
    r_lo = oracle.clip_ratios(g_lo, nb)
    r_hi = oracle.clip_ratios(g_hi, nb)
    ofmt = "e4m3" if fmt == "mxfp8" else "e2m1"
    oc, os_, bad = oracle.quantize(y_gpu.reshape(T * H, D), r_lo, r_hi, fmt=ofmt)
    assert bad == 0
    oc, os_ = oc.reshape(T, H, D), os_.reshape(T, H, nb)
    codes, scales = _kv_host(cache, fmt)
    for t in range(T):
        if slots[t] >= 0:
            assert np.array_equal(codes[slots[t]], oc[t]), t
            assert np.array_equal(scales[slots[t]], os_[t]), t
    untouched = np.setdiff1d(np.arange(S), slots[slots >= 0])
    raw = cache.codes.cpu().numpy().reshape(S, -1)
    assert np.all(raw[untouched] == 0x5A)
    assert np.all(scales[untouched] == 0xA5)
    assert bat.bat_device_error() == 0


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
@pytest.mark.parametrize("D,s", [(128, 8), (96, 4), (256, 16)])
def test_kv_dequantize_parity(bat, fmt, D, s):
    T, H, S = 24, 4, 32
    kv, A, B, g_lo, g_hi, slots, cache, _, _ = _kv_case(bat, T, H, D, S, fmt, s=s, seed=7)
    read = np.array([sl for sl in slots if sl >= 0] + [slots[slots >= 0][0]], np.int64)
    rd = torch.from_numpy(read).cuda()
    ofmt = "e4m3" if fmt == "mxfp8" else "e2m1"
    codes, scales = _kv_host(cache, fmt)
    # values as stored: exact (fp32 of the fp64 value)
    v = bat.bat_kv_dequantize(cache, rd).cpu().numpy()
    ref = oracle.kv_dequantize(codes, scales, read, ofmt)
    assert np.array_equal(v, ref.astype(np.float32))
    vb = bat.bat_kv_dequantize(cache, rd, out_dtype=torch.bfloat16).float().cpu().numpy()
    assert np.array_equal(vb, torch.from_numpy(v).to(torch.bfloat16).float().numpy())
    # through the inverse factors: back to K / V up to the quantization error
    Ai = oracle.inverse(A.astype(np.float64)).astype(np.float32)
    Bi = np.stack([oracle.inverse(b.astype(np.float64)) for b in B]).astype(np.float32)
    w = bat.bat_kv_dequantize(cache, rd, _dev_f32(Ai), _dev_f32(Bi)).cpu().numpy()
    refw = oracle.kv_dequantize(codes, scales, read, ofmt, Ai, Bi)
    _check_transform(w.reshape(-1, D), refw.reshape(-1, D))
    assert bat.bat_device_error() == 0


def test_kv_bad_slot_is_skipped_and_reported(bat):
    T, H, D, S = 3, 2, 64, 4
    kv = _dev_bf16(wl.random_bf16((T, H, D), seed=1))
    A, B, _, _ = wl.random_factors(D // 32, seed=2)
    cache = bat.KVCache.empty(S, H, D, "mxfp8")
    cache.codes.fill_(0x5A)
    slots = torch.tensor([0, S + 5, 2], dtype=torch.int64, device="cuda")
    bat.bat_kv_quantize(kv, _dev_f32(A), _dev_f32(B), slots, cache)
    torch.cuda.synchronize()
    assert bat.bat_device_error() != 0
    assert bat.bat_device_error() == 0  # read and cleared
    raw = cache.codes.cpu().numpy().reshape(S, -1)
    assert np.all(raw[1] == 0x5A) and np.all(raw[3] == 0x5A)
    out = bat.bat_kv_dequantize(cache, torch.tensor([1, -1, S], dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert bat.bat_device_error() != 0
    assert torch.all(out[1:] == 0)


def test_kv_bad_slot_prefill_path(bat):
    T, H, D, S = 1024, 8, 128, 1100
    kv = _dev_bf16(wl.random_bf16((T, H, D), seed=3))
    A, B, _, _ = wl.random_factors(D // 32, seed=4)
    cache = bat.KVCache.empty(S, H, D, "mxfp4")
    cache.codes.fill_(0x5A)
    sl = np.arange(T, dtype=np.int64)
    sl[5] = S + 1
    bat.bat_kv_quantize(kv, _dev_f32(A), _dev_f32(B), torch.from_numpy(sl).cuda(), cache)
    torch.cuda.synchronize()
    assert bat.bat_device_error() != 0
    raw = cache.codes.cpu().numpy().reshape(S, -1)
    assert np.all(raw[5] == 0x5A) and np.all(raw[T:] == 0x5A)
    assert not np.all(raw[4] == 0x5A)


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
def test_kv_prefill_size(bat, fmt):
    """A 4096-token prefill of 8 KV heads x 128 (Qwen3-8B-like), checked on sampled tokens."""
    T, H, D = 4096, 8, 128
    kv, A, B, g_lo, g_hi, slots, cache, y_gpu, _ = _kv_case(bat, T, H, D, T, fmt, seed=11)
    pick = _sample(T, 64, 5)
    nb = D // 32
    _check_transform(y_gpu[pick].reshape(-1, D), oracle.transform(kv[pick].reshape(-1, D), A, B))
    ofmt = "e4m3" if fmt == "mxfp8" else "e2m1"
    oc, os_, _ = oracle.quantize(y_gpu[pick].reshape(-1, D), oracle.clip_ratios(g_lo, nb),
                                 oracle.clip_ratios(g_hi, nb), fmt=ofmt)
    oc, os_ = oc.reshape(len(pick), H, D), os_.reshape(len(pick), H, nb)
    codes, scales = _kv_host(cache, fmt)
    for i, t in enumerate(pick):
        if slots[t] >= 0:
            assert np.array_equal(codes[slots[t]], oc[i]) and np.array_equal(scales[slots[t]], os_[i])
    assert bat.bat_device_error() == 0


def test_split_k_is_deterministic(bat):
    """The decode shape runs split-K over clusters; partials are summed in a fixed order."""
    M, N, K = 16, 6144, 4096
    X = wl.random_bf16((M, K), seed=21, scale=2.0)
    W = wl.random_bf16((N, K), seed=22, scale=0.02)
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=23)
    Ad, Bd = _dev_f32(A), _dev_f32(B)
    Xq = bat.bat_quantize_act(_dev_bf16(X), Ad, Bd, _dev_f32(g_lo), _dev_f32(g_hi))
    Wq = bat.bat_prepare_weight(_dev_bf16(W), Ad, Bd)
    ys = [bat.bat_mxfp4_gemm(Xq, Wq, out_dtype=torch.float32) for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0], y) for y in ys[1:])
    assert bat.bat_device_error() == 0


@pytest.mark.parametrize("M,N,K,clip", [(16, 6144, 4096, True), (1, 256, 2048, True),
                                        (16, 520, 1024, False), (7, 1000, 4128, True),
                                        (64, 520, 1024, True), (33, 264, 12288, True)])
def test_linear_at_decode_sizes_equals_two_calls(bat, M, N, K, clip):
    """bat_linear and bat_linear_noalloc at decode sizes (row quantizer, split-K GEMM)
    equal bat_quantize_act followed by bat_mxfp4_gemm bit for bit."""
    X = wl.random_bf16((M, K), seed=M + K, scale=3.0)
    W = wl.random_bf16((N, K), seed=N + K, scale=0.02)
    A, B, g_lo, g_hi = wl.random_factors(K // 32, seed=K + 9)
    Xd, Ad, Bd = _dev_bf16(X), _dev_f32(A), _dev_f32(B)
    gl = _dev_f32(g_lo) if clip else None
    gh = _dev_f32(g_hi) if clip else None
    Wq = bat.bat_prepare_weight(_dev_bf16(W), Ad, Bd)
    for dt in (torch.float32, torch.bfloat16):
        Y = bat.bat_linear(X=Xd, Wq=Wq, A=Ad, B=Bd, g_lo=gl, g_hi=gh, out_dtype=dt)
        Xq = bat.bat_quantize_act(Xd, Ad, Bd, gl, gh)
        Y2 = bat.bat_mxfp4_gemm(Xq, Wq, out_dtype=dt)
        Y3 = bat.bat_linear_noalloc(Xd, Wq, Ad, Bd, gl, gh, out_dtype=dt)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y2)
        assert torch.equal(Y3, Y2)
    assert bat.bat_device_error() == 0


def test_bounded_wait_reports_and_returns(bat):
    """A wait on a barrier nothing arrives on runs out after its limit, sets the device
    error word and returns; the context stays usable (a later call works)."""
    assert bat.bat_device_error() == 0
    assert bat.bat_selftest_bounded_wait(20_000_000) == 1
    assert bat.bat_device_error() != 0
    assert bat.bat_device_error() == 0
    r = bat.bat_clip_ratios(None, 4)
    torch.cuda.synchronize()
    assert torch.all(r == 1.0)

"""BATQuant W4A4 (MXFP4) linear layer for NVIDIA B200 (sm_100a).

Thin Python binding over the C-ABI in ``include/bat.h`` (``libbat.so``, built
in-tree by ``w4a4_bit_gemm_b200.build``). Every function here only marshals
torch tensors into pointers and sizes; all arithmetic runs in the library's
CUDA kernels. There is no CPU fallback: if the library cannot be loaded the
calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbat.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "bat.h")

BAT_OUT_BF16 = 0
BAT_OUT_F32 = 1

_STATUS = {
    0: "BAT_OK", 1: "BAT_ERR_INVALID_ARG", 2: "BAT_ERR_SHAPE", 3: "BAT_ERR_ALIGN",
    4: "BAT_ERR_SINGULAR", 5: "BAT_ERR_CUDA", 6: "BAT_ERR_UNSUPPORTED", 7: "BAT_ERR_WORKSPACE",
    8: "BAT_ERR_DEVICE",
}


class BatError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}")


class MXFP4Struct(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("k", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load ``libbat.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run w4a4_bit_gemm_b200.build.build() first")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    SP = ctypes.POINTER(MXFP4Struct)
    sig = {
        "bat_mxfp4_codes_bytes": (ctypes.c_size_t, [I64, I64]),
        "bat_mxfp4_scales_bytes": (ctypes.c_size_t, [I64, I64]),
        "bat_status_string": (ctypes.c_char_p, [S]),
        "bat_version": (S, []),
        "bat_quantize_act": (S, [P, I64, I64, P, P, P, P, SP, P]),
        "bat_quantize_act_trace": (S, [P, I64, I64, P, P, P, P, SP, P, P]),
        "bat_clip_ratios": (S, [P, I64, P, P]),
        "bat_e2m1_encode": (S, [P, I64, P, P]),
        "bat_prepare_weight": (S, [P, I64, I64, P, P, P, P, SP, P, P]),
        "bat_quantize_act_gpk": (S, [P, I64, I64, P, S, P, P, P, SP, P, P]),
        "bat_prepare_weight_gpk": (S, [P, I64, I64, P, S, P, P, P, SP, P, P]),
        "bat_block_hadamard_factors": (S, [S, I64, P, P]),
        "bat_mxfp8_codes_bytes": (ctypes.c_size_t, [I64, I64]),
        "bat_quantize_act_mxfp8": (S, [P, I64, I64, P, S, P, P, P, SP, P, P]),
        "bat_e4m3_encode": (S, [P, I64, P, P]),
        "bat_w4a8_gemm": (S, [SP, SP, P, S, P]),
        "bat_kv_codes_bytes": (ctypes.c_size_t, [I64, I64, I64, S]),
        "bat_kv_scales_bytes": (ctypes.c_size_t, [I64, I64, I64]),
        "bat_kv_quantize": (S, [P, I64, I64, I64, P, S, P, P, P, P, S, P, P, I64, P, P]),
        "bat_kv_dequantize": (S, [P, P, I64, I64, I64, S, P, I64, P, S, P, P, S, P]),
        "bat_selftest_bounded_wait": (S, [ctypes.c_uint64, P, P]),
        "bat_mxfp4_gemm": (S, [SP, SP, P, S, P]),
        "bat_linear_workspace_bytes": (ctypes.c_size_t, [I64, I64]),
        "bat_linear": (S, [P, I64, SP, P, P, P, P, P, S, P, ctypes.c_size_t, S, P]),
        "bat_linear_noalloc": (S, [P, I64, SP, P, P, P, P, P, S, P]),
        "bat_device_error": (S, []),
        "bat_last_cuda_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def declared_functions() -> list[str]:
    """Names of the functions ``include/bat.h`` declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bat_[a-z0-9_]+)\s*\(", text)))


# ---------------------------------------------------------------- marshalling helpers
def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# The library takes device pointers only: every tensor handed to it must live in GPU memory.
_DEVICE_TYPE = "cuda"


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, shape=None, device=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != _DEVICE_TYPE:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}; every tensor of the call must be on {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _need_bytes(t: torch.Tensor, name: str, nbytes: int, device) -> torch.Tensor:
    """A caller-supplied byte buffer the kernels write or read: large enough for its shape."""
    _need(t, torch.uint8, name, device=device)
    if t.numel() < nbytes:
        raise ValueError(f"{name} holds {t.numel()} bytes; {nbytes} are needed")
    return t


def _on_device(dev: torch.device, stream) -> None:
    """The kernels run on the current device, on `stream`: the tensors must live there."""
    if dev.type == "cuda" and dev.index is not None and dev.index != torch.cuda.current_device():
        raise ValueError(f"the tensors are on {dev} but the current device is "
                         f"cuda:{torch.cuda.current_device()}; call under torch.cuda.device({dev})")
    if stream is not None and getattr(stream, "device", dev) != dev:
        raise ValueError(f"the stream belongs to {stream.device}, the tensors to {dev}")


def _check(status: int, where: str) -> None:
    if status != 0:
        err = BatError(status, where)
        if status == 5:  # BAT_ERR_CUDA: attach the CUDA error text
            err.args = (f"{err.args[0]} ({lib().bat_last_cuda_error().decode()})",)
        raise err


@dataclass
class MXFP4:
    """An MXFP4 matrix: packed E2M1 codes [rows][k/2] and tiled UE8M0 scales."""
    codes: torch.Tensor
    scales: torch.Tensor
    rows: int
    k: int

    @staticmethod
    def empty(rows: int, k: int, device="cuda") -> "MXFP4":
        cb = bat_mxfp4_codes_bytes(rows, k)
        sb = bat_mxfp4_scales_bytes(rows, k)
        if cb == 0 or sb == 0:
            raise ValueError(f"invalid MXFP4 shape rows={rows} k={k}")
        return MXFP4(torch.empty(cb, dtype=torch.uint8, device=device),
                     torch.empty(sb, dtype=torch.uint8, device=device), rows, k)

    def struct(self) -> MXFP4Struct:
        return MXFP4Struct(self.codes.data_ptr(), self.scales.data_ptr(), self.rows, self.k)

    def check(self, name: str, device) -> "MXFP4":
        """Both buffers on `device` and large enough for rows x k (before any launch)."""
        _need_bytes(self.codes, f"{name}.codes", bat_mxfp4_codes_bytes(self.rows, self.k), device)
        _need_bytes(self.scales, f"{name}.scales", bat_mxfp4_scales_bytes(self.rows, self.k), device)
        return self


@dataclass
class MXFP8:
    """An MXFP8 matrix: E4M3 codes [rows][k] (one byte each) and tiled UE8M0 scales."""
    codes: torch.Tensor
    scales: torch.Tensor
    rows: int
    k: int

    @staticmethod
    def empty(rows: int, k: int, device="cuda") -> "MXFP8":
        cb = bat_mxfp8_codes_bytes(rows, k)
        sb = bat_mxfp4_scales_bytes(rows, k)
        if cb == 0 or sb == 0:
            raise ValueError(f"invalid MXFP8 shape rows={rows} k={k}")
        return MXFP8(torch.empty(cb, dtype=torch.uint8, device=device),
                     torch.empty(sb, dtype=torch.uint8, device=device), rows, k)

    def struct(self) -> MXFP4Struct:
        return MXFP4Struct(self.codes.data_ptr(), self.scales.data_ptr(), self.rows, self.k)

    def check(self, name: str, device) -> "MXFP8":
        _need_bytes(self.codes, f"{name}.codes", bat_mxfp8_codes_bytes(self.rows, self.k), device)
        _need_bytes(self.scales, f"{name}.scales", bat_mxfp4_scales_bytes(self.rows, self.k), device)
        return self


# ---------------------------------------------------------------- C-ABI wrappers
def bat_mxfp8_codes_bytes(rows: int, k: int) -> int:
    return lib().bat_mxfp8_codes_bytes(rows, k)



def bat_mxfp4_codes_bytes(rows: int, k: int) -> int:
    return lib().bat_mxfp4_codes_bytes(rows, k)


def bat_mxfp4_scales_bytes(rows: int, k: int) -> int:
    return lib().bat_mxfp4_scales_bytes(rows, k)


def bat_status_string(status: int) -> str:
    return lib().bat_status_string(status).decode()


def bat_version() -> int:
    return lib().bat_version()


def _act_args(X, A, B, g_lo, g_hi):
    _need(X, torch.bfloat16, "X")
    M, K = X.shape
    dev = X.device
    _need(A, torch.float32, "A", (8, 8), dev)
    _need(B, torch.float32, "B", (K // 32, 4, 4), dev)
    _clip_args(g_lo, g_hi, K // 32, dev)
    return M, K


def _clip_args(g_lo, g_hi, nb: int, dev, prefix: str = "g", rows=None):
    if (g_lo is None) != (g_hi is None):
        raise ValueError(f"{prefix}_lo and {prefix}_hi must both be given or both be None")
    if g_lo is not None:
        shape = (nb,) if rows is None else (rows, nb)
        _need(g_lo, torch.float32, f"{prefix}_lo", shape, dev)
        _need(g_hi, torch.float32, f"{prefix}_hi", shape, dev)


def bat_quantize_act(X, A, B, g_lo=None, g_hi=None, Xq: Optional[MXFP4] = None, stream=None) -> MXFP4:
    M, K = _act_args(X, A, B, g_lo, g_hi)
    Xq = (MXFP4.empty(M, K, X.device) if Xq is None else Xq).check("Xq", X.device)
    _on_device(X.device, stream)
    st = Xq.struct()
    _check(lib().bat_quantize_act(_ptr(X), M, K, _ptr(A), _ptr(B), _ptr(g_lo), _ptr(g_hi),
                                  ctypes.byref(st), _stream(stream)), "bat_quantize_act")
    return Xq


def bat_quantize_act_trace(X, A, B, g_lo=None, g_hi=None, Xq: Optional[MXFP4] = None,
                           y_out: Optional[torch.Tensor] = None, stream=None):
    M, K = _act_args(X, A, B, g_lo, g_hi)
    Xq = (MXFP4.empty(M, K, X.device) if Xq is None else Xq).check("Xq", X.device)
    y_out = torch.empty(M, K, dtype=torch.float32, device=X.device) if y_out is None else y_out
    _need(y_out, torch.float32, "y_out", (M, K), X.device)
    _on_device(X.device, stream)
    st = Xq.struct()
    _check(lib().bat_quantize_act_trace(_ptr(X), M, K, _ptr(A), _ptr(B), _ptr(g_lo), _ptr(g_hi),
                                        ctypes.byref(st), _ptr(y_out), _stream(stream)),
           "bat_quantize_act_trace")
    return Xq, y_out


def bat_clip_ratios(g: Optional[torch.Tensor], n: Optional[int] = None, r=None, stream=None):
    if g is not None:
        _need(g, torch.float32, "g")
        n = g.numel()
    dev = g.device if g is not None else (r.device if isinstance(r, torch.Tensor) else
                                          torch.device("cuda", torch.cuda.current_device()))
    r = torch.empty(n, dtype=torch.float32, device=dev) if r is None else r
    _need(r, torch.float32, "r", None, dev)
    if r.numel() < n:
        raise ValueError(f"r holds {r.numel()} values; {n} are needed")
    _on_device(dev, stream)
    _check(lib().bat_clip_ratios(_ptr(g), n, _ptr(r), _stream(stream)), "bat_clip_ratios")
    return r


def bat_e2m1_encode(v: torch.Tensor, codes=None, stream=None) -> torch.Tensor:
    _need(v, torch.float32, "v")
    codes = torch.empty(v.numel(), dtype=torch.uint8, device=v.device) if codes is None else codes
    _need_bytes(codes, "codes", v.numel(), v.device)
    _on_device(v.device, stream)
    _check(lib().bat_e2m1_encode(_ptr(v), v.numel(), _ptr(codes), _stream(stream)), "bat_e2m1_encode")
    return codes


def bat_prepare_weight(W, A, B, gw_lo=None, gw_hi=None, Wq: Optional[MXFP4] = None,
                       wt_out: Optional[torch.Tensor] = None, stream=None) -> MXFP4:
    _need(W, torch.bfloat16, "W")
    N, K = W.shape
    dev = W.device
    _need(A, torch.float32, "A", (8, 8), dev)
    _need(B, torch.float32, "B", (K // 32, 4, 4), dev)
    _clip_args(gw_lo, gw_hi, K // 32, dev, "gw", rows=N)
    if wt_out is not None:
        _need(wt_out, torch.float32, "wt_out", (N, K), dev)
    Wq = (MXFP4.empty(N, K, dev) if Wq is None else Wq).check("Wq", dev)
    _on_device(dev, stream)
    st = Wq.struct()
    _check(lib().bat_prepare_weight(_ptr(W), N, K, _ptr(A), _ptr(B), _ptr(gw_lo), _ptr(gw_hi),
                                    ctypes.byref(st), _ptr(wt_out), _stream(stream)),
           "bat_prepare_weight")
    return Wq


def _gpk_factors(A, B, K, dev=None):
    s = A.shape[0] if isinstance(A, torch.Tensor) and A.dim() == 2 else 0
    t = 32 // s if s else 0
    _need(A, torch.float32, "A", (s, s), dev)
    _need(B, torch.float32, "B", (K // 32, t, t), dev)
    return s


def bat_quantize_act_gpk(X, A, B, g_lo=None, g_hi=None, Xq: Optional[MXFP4] = None,
                         y_out: Optional[torch.Tensor] = None, stream=None) -> MXFP4:
    """Activation side with an s x s shared factor A and (32/s) x (32/s) private B_b."""
    _need(X, torch.bfloat16, "X")
    M, K = X.shape
    dev = X.device
    s = _gpk_factors(A, B, K, dev)
    _clip_args(g_lo, g_hi, K // 32, dev)
    if y_out is not None:
        _need(y_out, torch.float32, "y_out", (M, K), dev)
    Xq = (MXFP4.empty(M, K, dev) if Xq is None else Xq).check("Xq", dev)
    _on_device(dev, stream)
    st = Xq.struct()
    _check(lib().bat_quantize_act_gpk(_ptr(X), M, K, _ptr(A), s, _ptr(B), _ptr(g_lo), _ptr(g_hi),
                                      ctypes.byref(st), _ptr(y_out), _stream(stream)),
           "bat_quantize_act_gpk")
    return Xq


def bat_prepare_weight_gpk(W, A, B, gw_lo=None, gw_hi=None, Wq: Optional[MXFP4] = None,
                           wt_out: Optional[torch.Tensor] = None, stream=None) -> MXFP4:
    """Weight side for the factor split of ``bat_quantize_act_gpk``."""
    _need(W, torch.bfloat16, "W")
    N, K = W.shape
    dev = W.device
    s = _gpk_factors(A, B, K, dev)
    _clip_args(gw_lo, gw_hi, K // 32, dev, "gw", rows=N)
    if wt_out is not None:
        _need(wt_out, torch.float32, "wt_out", (N, K), dev)
    Wq = (MXFP4.empty(N, K, dev) if Wq is None else Wq).check("Wq", dev)
    _on_device(dev, stream)
    st = Wq.struct()
    _check(lib().bat_prepare_weight_gpk(_ptr(W), N, K, _ptr(A), s, _ptr(B), _ptr(gw_lo),
                                        _ptr(gw_hi), ctypes.byref(st), _ptr(wt_out),
                                        _stream(stream)), "bat_prepare_weight_gpk")
    return Wq


def bat_block_hadamard_factors(shared: int, nb: int):
    """Host (CPU) fp32 factors A = H_s/sqrt(s), B_b = H_t/sqrt(t) of the block Hadamard rotation."""
    t = 32 // shared if shared in (1, 2, 4, 8, 16, 32) else 1
    A = torch.empty(shared, shared, dtype=torch.float32) if shared > 0 else torch.empty(1)
    B = torch.empty(max(nb, 1), t, t, dtype=torch.float32)
    _check(lib().bat_block_hadamard_factors(shared, nb, _ptr(A), _ptr(B)),
           "bat_block_hadamard_factors")
    return A, B


def _out_code(out_dtype: torch.dtype) -> int:
    if out_dtype == torch.bfloat16:
        return BAT_OUT_BF16
    if out_dtype == torch.float32:
        return BAT_OUT_F32
    raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")


def bat_mxfp4_gemm(Xq: MXFP4, Wq: MXFP4, Y: Optional[torch.Tensor] = None,
                   out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    code = _out_code(out_dtype)
    dev = Xq.codes.device
    Xq.check("Xq", dev)
    Wq.check("Wq", dev)
    Y = torch.empty(Xq.rows, Wq.rows, dtype=out_dtype, device=dev) if Y is None else Y
    _need(Y, out_dtype, "Y", (Xq.rows, Wq.rows), dev)
    _on_device(dev, stream)
    a, b = Xq.struct(), Wq.struct()
    _check(lib().bat_mxfp4_gemm(ctypes.byref(a), ctypes.byref(b), _ptr(Y), code, _stream(stream)),
           "bat_mxfp4_gemm")
    return Y


def bat_quantize_act_mxfp8(X, A, B, g_lo=None, g_hi=None, Xq: Optional[MXFP8] = None,
                           y_out: Optional[torch.Tensor] = None, stream=None) -> MXFP8:
    """W4A8 activation side: transform (any split of A, B), clip, MXFP8 (E4M3) quantize."""
    _need(X, torch.bfloat16, "X")
    M, K = X.shape
    dev = X.device
    s = _gpk_factors(A, B, K, dev)
    _clip_args(g_lo, g_hi, K // 32, dev)
    if y_out is not None:
        _need(y_out, torch.float32, "y_out", (M, K), dev)
    Xq = (MXFP8.empty(M, K, dev) if Xq is None else Xq).check("Xq", dev)
    _on_device(dev, stream)
    st = Xq.struct()
    _check(lib().bat_quantize_act_mxfp8(_ptr(X), M, K, _ptr(A), s, _ptr(B), _ptr(g_lo),
                                        _ptr(g_hi), ctypes.byref(st), _ptr(y_out),
                                        _stream(stream)), "bat_quantize_act_mxfp8")
    return Xq


def bat_e4m3_encode(v: torch.Tensor, codes=None, stream=None) -> torch.Tensor:
    _need(v, torch.float32, "v")
    codes = torch.empty(v.numel(), dtype=torch.uint8, device=v.device) if codes is None else codes
    _need_bytes(codes, "codes", v.numel(), v.device)
    _on_device(v.device, stream)
    _check(lib().bat_e4m3_encode(_ptr(v), v.numel(), _ptr(codes), _stream(stream)), "bat_e4m3_encode")
    return codes


def bat_w4a8_gemm(Xq: MXFP8, Wq: MXFP4, Y: Optional[torch.Tensor] = None,
                  out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    code = _out_code(out_dtype)
    dev = Xq.codes.device
    Xq.check("Xq", dev)
    Wq.check("Wq", dev)
    Y = torch.empty(Xq.rows, Wq.rows, dtype=out_dtype, device=dev) if Y is None else Y
    _need(Y, out_dtype, "Y", (Xq.rows, Wq.rows), dev)
    _on_device(dev, stream)
    a, b = Xq.struct(), Wq.struct()
    _check(lib().bat_w4a8_gemm(ctypes.byref(a), ctypes.byref(b), _ptr(Y), code, _stream(stream)),
           "bat_w4a8_gemm")
    return Y


def bat_linear_workspace_bytes(M: int, K: int) -> int:
    return lib().bat_linear_workspace_bytes(M, K)


def bat_linear(X, Wq: MXFP4, A, B, g_lo=None, g_hi=None, Y: Optional[torch.Tensor] = None,
               out_dtype: torch.dtype = torch.bfloat16, workspace: Optional[torch.Tensor] = None,
               stream=None, fused: bool = False) -> torch.Tensor:
    M, K = _act_args(X, A, B, g_lo, g_hi)
    code = _out_code(out_dtype)
    dev = X.device
    if Wq.k != K:
        raise ValueError(f"Wq has k={Wq.k} but X has K={K}")
    Wq.check("Wq", dev)
    Y = torch.empty(M, Wq.rows, dtype=out_dtype, device=dev) if Y is None else Y
    _need(Y, out_dtype, "Y", (M, Wq.rows), dev)
    need = bat_linear_workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _need(workspace, torch.uint8, "workspace", None, dev)
    _on_device(dev, stream)
    b = Wq.struct()
    _check(lib().bat_linear(_ptr(X), M, ctypes.byref(b), _ptr(A), _ptr(B), _ptr(g_lo), _ptr(g_hi),
                            _ptr(Y), code, _ptr(workspace), workspace.numel(), 1 if fused else 0,
                            _stream(stream)),
           "bat_linear")
    return Y


NOALLOC_SCRATCH_BYTES = 8 << 20  # BAT_NOALLOC_SCRATCH_BYTES in include/bat.h


def bat_linear_noalloc(X, Wq: MXFP4, A, B, g_lo=None, g_hi=None, Y: Optional[torch.Tensor] = None,
                       out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """bat_linear without a workspace: the library's own static device scratch holds
    the quantized activations (for callers that cannot allocate device memory)."""
    M, K = _act_args(X, A, B, g_lo, g_hi)
    code = _out_code(out_dtype)
    dev = X.device
    if Wq.k != K:
        raise ValueError(f"Wq has k={Wq.k} but X has K={K}")
    Wq.check("Wq", dev)
    Y = torch.empty(M, Wq.rows, dtype=out_dtype, device=dev) if Y is None else Y
    _need(Y, out_dtype, "Y", (M, Wq.rows), dev)
    _on_device(dev, stream)
    b = Wq.struct()
    _check(lib().bat_linear_noalloc(_ptr(X), M, ctypes.byref(b), _ptr(A), _ptr(B), _ptr(g_lo),
                                    _ptr(g_hi), _ptr(Y), code, _stream(stream)),
           "bat_linear_noalloc")
    return Y


def bat_device_error() -> int:
    return lib().bat_device_error()


# ---------------------------------------------------------------- KV cache
BAT_KV_MXFP8, BAT_KV_MXFP4 = 0, 1
_KV_FMT = {"mxfp8": BAT_KV_MXFP8, "mxfp4": BAT_KV_MXFP4}


@dataclass
class KVCache:
    """One K (or V) cache: codes [S][H][D] E4M3 or [S][H][D/2] packed E2M1, scales [S][H][D/32]."""
    codes: torch.Tensor
    scales: torch.Tensor
    num_slots: int
    H: int
    D: int
    fmt: str

    @staticmethod
    def empty(num_slots: int, H: int, D: int, fmt: str = "mxfp8", device="cuda") -> "KVCache":
        f = _KV_FMT[fmt]
        cb = lib().bat_kv_codes_bytes(num_slots, H, D, f)
        sb = lib().bat_kv_scales_bytes(num_slots, H, D)
        if cb == 0 or sb == 0:
            raise ValueError(f"invalid KV cache shape {num_slots}x{H}x{D}")
        return KVCache(torch.zeros(cb, dtype=torch.uint8, device=device),
                       torch.zeros(sb, dtype=torch.uint8, device=device), num_slots, H, D, fmt)

    def check(self, device) -> "KVCache":
        """Both buffers on `device` and large enough for num_slots x H x D (before any launch)."""
        if self.fmt not in _KV_FMT:
            raise ValueError(f"unknown KV format {self.fmt!r}")
        f = _KV_FMT[self.fmt]
        _need_bytes(self.codes, "cache.codes",
                    lib().bat_kv_codes_bytes(self.num_slots, self.H, self.D, f), device)
        _need_bytes(self.scales, "cache.scales",
                    lib().bat_kv_scales_bytes(self.num_slots, self.H, self.D), device)
        return self


def bat_kv_quantize(kv, A, B, slots, cache: KVCache, g_lo=None, g_hi=None,
                    y_out: Optional[torch.Tensor] = None, stream=None) -> KVCache:
    """Transform, clip and quantize kv [T][H][D] (bf16) into cache rows slots[t] (-1 skips)."""
    _need(kv, torch.bfloat16, "kv")
    T, H, D = kv.shape
    dev = kv.device
    s = _gpk_factors(A, B, D, dev)
    _need(slots, torch.int64, "slots", (T,), dev)
    _clip_args(g_lo, g_hi, D // 32, dev)
    if y_out is not None:
        _need(y_out, torch.float32, "y_out", (T, H, D), dev)
    if cache.H != H or cache.D != D:
        raise ValueError("cache shape does not match kv")
    cache.check(dev)
    _on_device(dev, stream)
    _check(lib().bat_kv_quantize(_ptr(kv), T, H, D, _ptr(A), s, _ptr(B), _ptr(g_lo), _ptr(g_hi),
                                 _ptr(slots), _KV_FMT[cache.fmt], _ptr(cache.codes),
                                 _ptr(cache.scales), cache.num_slots, _ptr(y_out),
                                 _stream(stream)), "bat_kv_quantize")
    return cache


def bat_kv_dequantize(cache: KVCache, slots, A=None, B=None, out: Optional[torch.Tensor] = None,
                      out_dtype: torch.dtype = torch.float32, stream=None) -> torch.Tensor:
    """Values of cache rows slots[t] as [T][H][D]; with A, B also multiplied by B_b (x) A."""
    dev = cache.codes.device
    cache.check(dev)
    _need(slots, torch.int64, "slots", None, dev)
    if slots.dim() != 1:
        raise ValueError("slots must be one-dimensional")
    T = slots.shape[0]
    s = 8
    if A is not None:
        s = _gpk_factors(A, B, cache.D, dev)
    code = _out_code(out_dtype)
    out = torch.empty(T, cache.H, cache.D, dtype=out_dtype, device=dev) if out is None else out
    _need(out, out_dtype, "out", (T, cache.H, cache.D), dev)
    _on_device(dev, stream)
    _check(lib().bat_kv_dequantize(_ptr(cache.codes), _ptr(cache.scales), cache.num_slots, cache.H,
                                   cache.D, _KV_FMT[cache.fmt], _ptr(slots), T, _ptr(A), s, _ptr(B),
                                   _ptr(out), code, _stream(stream)), "bat_kv_dequantize")
    return out


def bat_selftest_bounded_wait(limit_ns: int = 50_000_000, stream=None) -> int:
    """Run the bounded-wait self-test; returns the device flag (1: the wait ran out)."""
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(lib().bat_selftest_bounded_wait(limit_ns, _ptr(flag), _stream(stream)),
           "bat_selftest_bounded_wait")
    return int(flag.item())

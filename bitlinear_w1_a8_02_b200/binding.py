"""Thin Python binding of ``libbitlinear.so`` (the C ABI in include/bitlinear.h).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels. torch supplies device memory and the current stream. If the
library is missing or fails to load, every call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear.so")

# bl_status values
BL_OK = 0
STATUS_NAMES = {
    0: "BL_OK", 1: "BL_ERR_NULL", 2: "BL_ERR_SHAPE", 3: "BL_ERR_ALIGN", 4: "BL_ERR_DTYPE",
    5: "BL_ERR_WORKSPACE", 6: "BL_ERR_UNSUPPORTED", 7: "BL_ERR_CUDA", 8: "BL_ERR_TIMEOUT",
    9: "BL_ERR_BAD_CODE",
}
BL_BF16, BL_FP32 = 0, 1
BL_OP_PACK, BL_OP_FORWARD, BL_OP_FFN, BL_OP_VALIDATE, BL_OP_FFN_TP_UP, BL_OP_FFN_TP_DOWN = 0, 1, 2, 3, 4, 5
BL_GEMV_AUTO, BL_GEMV_STREAM, BL_GEMV_TENSOR, BL_GEMV_LUT = 0, 1, 2, 3

# Every symbol include/bitlinear.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int64
_S = ctypes.c_size_t
_ST = ctypes.c_int
SIGNATURES = {
    "bitlinear_status_string": (ctypes.c_char_p, [_ST]),
    "bitlinear_workspace_bytes": (_S, [ctypes.c_int, _I, _I, _I]),
    "bitlinear_pack_weights": (_ST, [_P, ctypes.c_int, _I, _I, _P, _P, _P, _S, _P]),
    "bitlinear_quant_act": (_ST, [_P, _I, _I, _P, _P, _P, _P]),
    "bitlinear_forward": (_ST, [_P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _S, _P]),
    "bitlinear_pack_weights_rowwise": (_ST, [_P, ctypes.c_int, _I, _I, _P, _P, _P]),
    "bitlinear_forward_rowwise": (_ST, [_P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _S, _P]),
    "bitlinear_forward_ex": (_ST, [_P, _P, _P, ctypes.c_int32, _I, _P, _I, ctypes.c_int32, _P, _P, _P, _P, _S,
                                   _P]),
    "bitlinear_ffn": (_ST, [_P, _P, _P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _S, _P]),
    "bitlinear_forward_noalloc": (_ST, [_P, _P, _I, _I, _P, _I, _P, _P, _P, _P]),
    "bitlinear_validate_packed": (_ST, [_P, _I, _I, _P, _P, _S, _P]),
    "bitlinear_get_device_error": (_ST, [_P]),
    "bitlinear_selftest_timeout": (_ST, [_I, _P]),
    "bitlinear_set_gemv_kernel": (ctypes.c_int, [ctypes.c_int]),
    "bitlinear_absmean_sum": (_ST, [_P, ctypes.c_int, _I, _I, _P, _P, _S, _P]),
    "bitlinear_pack_weights_global": (_ST, [_P, ctypes.c_int, _I, _I, _P, _I, _P, _P, _P]),
    "bitlinear_ffn_tp_up": (_ST, [_P, _P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _S, _P]),
    "bitlinear_ffn_tp_down": (_ST, [_P, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _S, _P]),
    "bitlinear_ffn_tp_finish": (_ST, [_P, _P, _P, _P, _P, _I, _I, _P]),
}


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} "
                         f"({lib().bitlinear_status_string(status).decode()})")


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python bitlinear_w1_a8_02_b200/build.py` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(st: int, where: str):
    if st != BL_OK:
        raise BitLinearError(st, where)


def _cuda(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def workspace_bytes(op: int, M: int, N: int, K: int) -> int:
    return int(lib().bitlinear_workspace_bytes(op, M, N, K))


class Workspace:
    """A reusable device workspace that grows on demand (one per device)."""

    def __init__(self):
        self._buf = {}

    def get(self, device: torch.device, nbytes: int) -> torch.Tensor:
        buf = self._buf.get(device)
        if buf is None or buf.numel() < nbytes:
            buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
            self._buf[device] = buf
        return buf


_WS = Workspace()


def pack_weights(W: torch.Tensor, ws: Optional[torch.Tensor] = None):
    """W [N, K] (bf16 or fp32, CUDA) -> (Wp [N, K/4] uint8, gamma [1] fp32)."""
    _cuda(W, "W")
    if W.dtype == torch.bfloat16:
        wdt = BL_BF16
    elif W.dtype == torch.float32:
        wdt = BL_FP32
    else:
        raise ValueError("W must be bf16 or fp32")
    N, K = W.shape
    Wp = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    need = workspace_bytes(BL_OP_PACK, 0, N, K)
    ws = _WS.get(W.device, need) if ws is None else ws
    st = lib().bitlinear_pack_weights(_ptr(W), wdt, N, K, _ptr(Wp), _ptr(gamma), _ptr(ws),
                                      ws.numel(), _stream(W.device))
    _check(st, "bitlinear_pack_weights")
    return Wp, gamma


def quant_act(x: torch.Tensor):
    """x [M, K] bf16 -> (xq int8 [M, K], scale fp32 [M], xsum int32 [M])."""
    _cuda(x, "x", torch.bfloat16)
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = torch.empty(M, dtype=torch.float32, device=x.device)
    xs = torch.empty(M, dtype=torch.int32, device=x.device)
    st = lib().bitlinear_quant_act(_ptr(x), M, K, _ptr(xq), _ptr(s), _ptr(xs), _stream(x.device))
    _check(st, "bitlinear_quant_act")
    return xq, s, xs


def forward(Wp: torch.Tensor, gamma: torch.Tensor, x: torch.Tensor,
            residual: Optional[torch.Tensor] = None, want_acc: bool = False,
            out: Optional[torch.Tensor] = None, acc: Optional[torch.Tensor] = None,
            ws: Optional[torch.Tensor] = None):
    """y = BitLinear(x) as bf16 [M, N]; with want_acc also the int32 accumulator."""
    _cuda(Wp, "Wp", torch.uint8)
    _cuda(x, "x", torch.bfloat16)
    N, KB = Wp.shape
    M, K = x.shape
    if K != 4 * KB:
        raise ValueError(f"x has K={K}, packed weights have K={4 * KB}")
    if residual is not None:
        _cuda(residual, "residual", torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    if want_acc and acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=x.device)
    need = workspace_bytes(BL_OP_FORWARD, M, N, K)
    ws = _WS.get(x.device, need) if ws is None else ws
    st = lib().bitlinear_forward(_ptr(Wp), _ptr(gamma), N, K, _ptr(x), M, _ptr(residual), _ptr(y),
                                 _ptr(acc), _ptr(ws), ws.numel(), _stream(x.device))
    _check(st, "bitlinear_forward")
    return (y, acc) if want_acc else y


def pack_weights_rowwise(W: torch.Tensor):
    """Per-row absmean variant: W [N, K] (bf16 or fp32, CUDA) -> (Wp uint8 [N, K/4], gammas fp32 [N])."""
    if W.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("W must be bf16 or fp32")
    _cuda(W, "W", W.dtype)
    N, K = W.shape
    Wp = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    gammas = torch.empty(N, dtype=torch.float32, device=W.device)
    st = lib().bitlinear_pack_weights_rowwise(_ptr(W), BL_FP32 if W.dtype == torch.float32 else BL_BF16, N, K,
                                              _ptr(Wp), _ptr(gammas), _stream(W.device))
    _check(st, "bitlinear_pack_weights_rowwise")
    return Wp, gammas


def forward_rowwise(Wp: torch.Tensor, gammas: torch.Tensor, x: torch.Tensor,
                    residual: Optional[torch.Tensor] = None, want_acc: bool = False,
                    out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """bitlinear_forward with one gamma per output row."""
    _cuda(Wp, "Wp", torch.uint8)
    _cuda(x, "x", torch.bfloat16)
    _cuda(gammas, "gammas", torch.float32)
    N, KB = Wp.shape
    M, K = x.shape
    if K != 4 * KB or gammas.numel() != N:
        raise ValueError("shapes of Wp, gammas and x do not match")
    if residual is not None:
        _cuda(residual, "residual", torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    acc = torch.empty((M, N), dtype=torch.int32, device=x.device) if want_acc else None
    need = workspace_bytes(BL_OP_FORWARD, M, N, K)
    ws = _WS.get(x.device, need) if ws is None else ws
    st = lib().bitlinear_forward_rowwise(_ptr(Wp), _ptr(gammas), N, K, _ptr(x), M, _ptr(residual), _ptr(y),
                                         _ptr(acc), _ptr(ws), ws.numel(), _stream(x.device))
    _check(st, "bitlinear_forward_rowwise")
    return (y, acc) if want_acc else y


def forward_ex(Wp: torch.Tensor, gammas: torch.Tensor, seg_rows, x: torch.Tensor, rmsnorm: bool = False,
               residual: Optional[torch.Tensor] = None, want_acc: bool = False,
               out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """Projections of x against row-stacked packed weights (segment i has
    seg_rows[i] rows and gamma gammas[i]), optionally after a unit-weight RMSNorm
    of x: bf16 [M, sum(seg_rows)] (and the int32 accumulator with want_acc)."""
    _cuda(Wp, "Wp", torch.uint8)
    _cuda(x, "x", torch.bfloat16)
    _cuda(gammas, "gammas", torch.float32)
    N, KB = Wp.shape
    M, K = x.shape
    rows = (ctypes.c_int64 * len(seg_rows))(*[int(r) for r in seg_rows])
    if sum(int(r) for r in seg_rows) != N:
        raise ValueError(f"segments cover {sum(seg_rows)} rows, packed weights have {N}")
    if K != 4 * KB:
        raise ValueError(f"x has K={K}, packed weights have K={4 * KB}")
    if residual is not None:
        _cuda(residual, "residual", torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else out
    acc = torch.empty((M, N), dtype=torch.int32, device=x.device) if want_acc else None
    need = workspace_bytes(BL_OP_FORWARD, M, N, K)
    ws = _WS.get(x.device, need) if ws is None else ws
    st = lib().bitlinear_forward_ex(_ptr(Wp), _ptr(gammas), rows, len(seg_rows), K, _ptr(x), M, int(bool(rmsnorm)),
                                    _ptr(residual), _ptr(y), _ptr(acc), _ptr(ws), ws.numel(), _stream(x.device))
    _check(st, "bitlinear_forward_ex")
    return (y, acc) if want_acc else y


def ffn(Wg, gg, Wu, gu, Wd, gd, x: torch.Tensor, residual: Optional[torch.Tensor] = None,
        out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """One FFN sub-layer (gate/up, ReLU^2, subln, requant, down, + residual)."""
    _cuda(x, "x", torch.bfloat16)
    M, d = x.shape
    f = Wg.shape[0]
    for t, name in ((Wg, "Wg"), (Wu, "Wu"), (Wd, "Wd")):
        _cuda(t, name, torch.uint8)
    if Wg.shape != (f, d // 4) or Wu.shape != (f, d // 4) or Wd.shape != (d, f // 4):
        raise ValueError("FFN weight shapes do not match x")
    if residual is not None:
        _cuda(residual, "residual", torch.bfloat16)
    y = torch.empty((M, d), dtype=torch.bfloat16, device=x.device) if out is None else out
    need = workspace_bytes(BL_OP_FFN, M, f, d)
    ws = _WS.get(x.device, need) if ws is None else ws
    st = lib().bitlinear_ffn(_ptr(Wg), _ptr(gg), _ptr(Wu), _ptr(gu), _ptr(Wd), _ptr(gd), d, f,
                             _ptr(x), M, _ptr(residual), _ptr(y), _ptr(ws), ws.numel(),
                             _stream(x.device))
    _check(st, "bitlinear_ffn")
    return y


def validate_packed(Wp: torch.Tensor) -> int:
    """Number of invalid (== 3) codes in Wp; synchronises the current stream."""
    _cuda(Wp, "Wp", torch.uint8)
    N, KB = Wp.shape
    ws = _WS.get(Wp.device, workspace_bytes(BL_OP_VALIDATE, 0, 0, 0))
    bad = ctypes.c_int64(0)
    st = lib().bitlinear_validate_packed(_ptr(Wp), N, 4 * KB, ctypes.byref(bad), _ptr(ws),
                                         ws.numel(), _stream(Wp.device))
    if st not in (BL_OK, 9):
        _check(st, "bitlinear_validate_packed")
    return int(bad.value)


def get_device_error(device=None) -> int:
    """Synchronise and return the pending device status (0 when clean)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return int(lib().bitlinear_get_device_error(_stream(device)))


def set_gemv_kernel(kind: int) -> int:
    """Process-wide choice of the M <= 16 kernel (BL_GEMV_*); returns the previous one."""
    prev = int(lib().bitlinear_set_gemv_kernel(int(kind)))
    if prev < 0:
        raise ValueError(f"unknown GEMV kernel {kind}")
    return prev


class gemv_kernel:
    """Context manager: run the enclosed calls with one M <= 16 kernel."""

    def __init__(self, kind: int):
        self.kind = kind
        self.prev = None

    def __enter__(self):
        self.prev = set_gemv_kernel(self.kind)
        return self

    def __exit__(self, *exc):
        set_gemv_kernel(self.prev)
        return False


# ----------------------------------------------------------------------------- tensor-parallel pieces

def _wdt(W: torch.Tensor) -> int:
    if W.dtype == torch.bfloat16:
        return BL_BF16
    if W.dtype == torch.float32:
        return BL_FP32
    raise ValueError("W must be bf16 or fp32")


def absmean_sum(W: torch.Tensor) -> torch.Tensor:
    """fp64 sum of |W| of one weight shard [N, K]: a device float64 tensor [1]."""
    _cuda(W, "W")
    N, K = W.shape
    out = torch.empty(1, dtype=torch.float64, device=W.device)
    ws = _WS.get(W.device, workspace_bytes(BL_OP_PACK, 0, N, K))
    st = lib().bitlinear_absmean_sum(_ptr(W), _wdt(W), N, K, _ptr(out), _ptr(ws), ws.numel(), _stream(W.device))
    _check(st, "bitlinear_absmean_sum")
    return out


def pack_weights_global(W: torch.Tensor, total_sum: torch.Tensor, total_count: int):
    """Pack a shard [N, K] with gamma = fp32(total_sum / total_count) of the whole
    tensor (total_sum: device float64 [1]) -> (Wp uint8 [N, K/4], gamma fp32 [1])."""
    _cuda(W, "W")
    _cuda(total_sum, "total_sum", torch.float64)
    N, K = W.shape
    Wp = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    st = lib().bitlinear_pack_weights_global(_ptr(W), _wdt(W), N, K, _ptr(total_sum), int(total_count), _ptr(Wp),
                                             _ptr(gamma), _stream(W.device))
    _check(st, "bitlinear_pack_weights_global")
    return Wp, gamma


def ffn_tp_up(Wg, gg, Wu, gu, x: torch.Tensor):
    """Rank-local gate/up of the FFN: (h fp32 [M, f_local], ss fp64 [M], hmax fp32 [M])."""
    _cuda(x, "x", torch.bfloat16)
    M, d = x.shape
    fl = Wg.shape[0]
    for t, name in ((Wg, "Wg"), (Wu, "Wu")):
        _cuda(t, name, torch.uint8)
    if Wg.shape != (fl, d // 4) or Wu.shape != (fl, d // 4):
        raise ValueError("gate / up shard shapes do not match x")
    h = torch.empty((M, fl), dtype=torch.float32, device=x.device)
    ss = torch.empty(M, dtype=torch.float64, device=x.device)
    hmax = torch.empty(M, dtype=torch.float32, device=x.device)
    ws = _WS.get(x.device, workspace_bytes(BL_OP_FFN_TP_UP, M, fl, d))
    st = lib().bitlinear_ffn_tp_up(_ptr(Wg), _ptr(gg), _ptr(Wu), _ptr(gu), d, fl, _ptr(x), M, _ptr(h), _ptr(ss),
                                   _ptr(hmax), _ptr(ws), ws.numel(), _stream(x.device))
    _check(st, "bitlinear_ffn_tp_up")
    return h, ss, hmax


def ffn_tp_down(Wd, h: torch.Tensor, ss_all: torch.Tensor, hmax_all: torch.Tensor, f_total: int):
    """Rank-local requantisation (global statistics) and partial down projection:
    (acc int32 [M, d], s2 fp32 [M])."""
    _cuda(Wd, "Wd", torch.uint8)
    _cuda(h, "h", torch.float32)
    _cuda(ss_all, "ss_all", torch.float64)
    _cuda(hmax_all, "hmax_all", torch.float32)
    M, fl = h.shape
    d = Wd.shape[0]
    if Wd.shape != (d, fl // 4):
        raise ValueError("down shard shape does not match h")
    acc = torch.empty((M, d), dtype=torch.int32, device=h.device)
    s2 = torch.empty(M, dtype=torch.float32, device=h.device)
    ws = _WS.get(h.device, workspace_bytes(BL_OP_FFN_TP_DOWN, M, d, fl))
    st = lib().bitlinear_ffn_tp_down(_ptr(Wd), d, fl, int(f_total), _ptr(h), M, _ptr(ss_all), _ptr(hmax_all),
                                     _ptr(acc), _ptr(s2), _ptr(ws), ws.numel(), _stream(h.device))
    _check(st, "bitlinear_ffn_tp_down")
    return acc, s2


def ffn_tp_finish(acc: torch.Tensor, gd, s2: torch.Tensor, residual: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None):
    """y = bf16([residual +] acc * (gd / s2)) on the accumulators summed over the ranks."""
    _cuda(acc, "acc", torch.int32)
    M, d = acc.shape
    if residual is not None:
        _cuda(residual, "residual", torch.bfloat16)
    y = torch.empty((M, d), dtype=torch.bfloat16, device=acc.device) if out is None else out
    st = lib().bitlinear_ffn_tp_finish(_ptr(acc), _ptr(gd), _ptr(s2), _ptr(residual), _ptr(y), M, d,
                                       _stream(acc.device))
    _check(st, "bitlinear_ffn_tp_finish")
    return y

"""CPU oracle for the BitLinear W1.58A8 forward of BitNet b1.58.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package. It shares no code with the
CUDA library: the arithmetic lives in ``bitlinear_oracle.c`` (plain C loops,
compiled with ``-ffp-contract=off``), and this module only marshals numpy arrays
into it. It never imports the product package.

Every function names the passage it follows in ``bitlinear_oracle.c``. Arrays
use numpy dtypes: bf16 tensors travel as their ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
          "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile ``bitlinear_oracle.c`` into ``liboracle.so`` (gcc) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _l():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int64
        F = ctypes.c_float
        sig = {
            "orc_set_threads": (ctypes.c_int, [ctypes.c_int]),
            "orc_bf16_to_f32": (F, [ctypes.c_uint16]),
            "orc_f32_to_bf16": (ctypes.c_uint16, [F]),
            "orc_bf16_to_f32_array": (None, [P, I, P]),
            "orc_f32_to_bf16_array": (None, [P, I, P]),
            "orc_absmean": (F, [P, I]),
            "orc_ternarize": (None, [P, I, F, P]),
            "orc_pack": (None, [P, I, I, P]),
            "orc_unpack": (I, [P, I, I, P]),
            "orc_pack_weights": (ctypes.c_int, [P, I, I, P, P]),
            "orc_quant_act": (None, [P, I, I, P, P, P]),
            "orc_int_gemm": (None, [P, P, I, I, I, P]),
            "orc_int_gemm_packed": (None, [P, P, I, I, I, P]),
            "orc_dequant": (None, [P, F, P, I, I, P, P, P]),
            "orc_forward": (ctypes.c_int, [P, F, I, I, P, I, P, P, P, P, P, P]),
            "orc_subln_rms": (F, [P, I, P]),
            "orc_relu2_gate": (F, [F, F]),
            "orc_ffn_layer": (ctypes.c_int, [P, F, P, F, P, F, I, I, P, I, P, P, P, P, P, P, P]),
            "orc_forward_ex": (ctypes.c_int, [P, P, P, I, I, P, I, I, P, P, P]),
            "orc_pack_weights_rowwise": (ctypes.c_int, [P, I, I, P, P]),
            "orc_absmean_sum": (ctypes.c_double, [P, I]),
            "orc_pack_weights_global": (ctypes.c_int, [P, I, I, ctypes.c_double, I, P, P]),
            "orc_ffn_tp_up": (ctypes.c_int, [P, F, P, F, I, I, P, I, P, P, P]),
            "orc_ffn_tp_down": (ctypes.c_int, [P, I, I, I, P, I, P, P, P, P]),
            "orc_forward_rowwise": (ctypes.c_int, [P, P, I, I, P, I, P, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- threads

def set_threads(n: int) -> int:
    """Threads of the oracle's OpenMP loops (0 leaves it unchanged); returns the
    count in effect. Results do not depend on it."""
    return int(_l().orc_set_threads(int(n)))


# --------------------------------------------------------------------------- bf16

def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    _l().orc_bf16_to_f32_array(_p(h), h.size, _p(out))
    return out


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    f = _c(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    _l().orc_f32_to_bf16_array(_p(f), f.size, _p(out))
    return out


# --------------------------------------------------------------------------- weights

def absmean(W: np.ndarray) -> np.float32:
    """gamma = mean |W| (fp64 sum, one rounding to fp32)."""
    W = _c(W, np.float32)
    return np.float32(_l().orc_absmean(_p(W), W.size))


def ternarize(W: np.ndarray, gamma) -> np.ndarray:
    """Wq = clip(rint(W / (gamma + 1e-5)), -1, 1) as int8."""
    W = _c(W, np.float32)
    q = np.empty(W.shape, np.int8)
    _l().orc_ternarize(_p(W), W.size, float(np.float32(gamma)), _p(q))
    return q


def pack(q: np.ndarray) -> np.ndarray:
    """[N, K] ternary int8 -> [N, K/4] uint8 (code q+1 at bits 2i of byte k//4)."""
    q = _c(q, np.int8)
    N, K = q.shape
    assert K % 4 == 0
    Wp = np.empty((N, K // 4), np.uint8)
    _l().orc_pack(_p(q), N, K, _p(Wp))
    return Wp


def unpack(Wp: np.ndarray, K: int):
    """[N, K/4] uint8 -> ([N, K] int8, number of invalid codes)."""
    Wp = _c(Wp, np.uint8)
    N = Wp.shape[0]
    assert Wp.shape[1] * 4 == K
    q = np.empty((N, K), np.int8)
    bad = _l().orc_unpack(_p(Wp), N, K, _p(q))
    return q, int(bad)


def pack_weights(W: np.ndarray):
    """Float weights [N, K] (fp32 or bf16 bits) -> (Wp [N, K/4] uint8, gamma fp32)."""
    if W.dtype == np.uint16:
        W = bf16_to_f32(W)
    W = _c(W, np.float32)
    N, K = W.shape
    Wp = np.empty((N, K // 4), np.uint8)
    g = np.zeros(1, np.float32)
    rc = _l().orc_pack_weights(_p(W), N, K, _p(Wp), _p(g))
    if rc != 0:
        raise MemoryError("oracle pack_weights failed")
    return Wp, np.float32(g[0])


# --------------------------------------------------------------------------- activations

def quant_act(x: np.ndarray):
    """x [M, K] (fp32, or bf16 bits) -> (xq int8 [M, K], s fp32 [M], xsum int32 [M])."""
    if x.dtype == np.uint16:
        x = bf16_to_f32(x)
    x = _c(x, np.float32)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    xs = np.empty(M, np.int32)
    _l().orc_quant_act(_p(x), M, K, _p(xq), _p(s), _p(xs))
    return xq, s, xs


# --------------------------------------------------------------------------- contraction

def int_gemm(q: np.ndarray, xq: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k q[n, k] * xq[m, k] (int32)."""
    q = _c(q, np.int8)
    xq = _c(xq, np.int8)
    N, K = q.shape
    M = xq.shape[0]
    assert xq.shape[1] == K
    acc = np.empty((M, N), np.int32)
    _l().orc_int_gemm(_p(q), _p(xq), M, N, K, _p(acc))
    return acc


def int_gemm_packed(Wp: np.ndarray, xq: np.ndarray) -> np.ndarray:
    Wp = _c(Wp, np.uint8)
    xq = _c(xq, np.int8)
    N = Wp.shape[0]
    M, K = xq.shape
    assert Wp.shape[1] * 4 == K
    acc = np.empty((M, N), np.int32)
    _l().orc_int_gemm_packed(_p(Wp), _p(xq), M, N, K, _p(acc))
    return acc


def dequant(acc: np.ndarray, gamma, s: np.ndarray, residual=None, want_f32=False):
    acc = _c(acc, np.int32)
    s = _c(s, np.float32)
    M, N = acc.shape
    res = None if residual is None else _c(residual, np.uint16)
    y = np.empty((M, N), np.uint16)
    y32 = np.empty((M, N), np.float32) if want_f32 else None
    _l().orc_dequant(_p(acc), float(np.float32(gamma)), _p(s), M, N, _p(res), _p(y), _p(y32))
    return (y, y32) if want_f32 else y


# --------------------------------------------------------------------------- forward / FFN

def forward(Wp: np.ndarray, gamma, x_bf16: np.ndarray, residual=None):
    """One BitLinear forward. Returns dict(y, acc, xq, s, xsum); y as bf16 bits."""
    Wp = _c(Wp, np.uint8)
    x = _c(x_bf16, np.uint16)
    N = Wp.shape[0]
    M, K = x.shape
    assert Wp.shape[1] * 4 == K
    res = None if residual is None else _c(residual, np.uint16)
    y = np.empty((M, N), np.uint16)
    acc = np.empty((M, N), np.int32)
    xq = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    xs = np.empty(M, np.int32)
    rc = _l().orc_forward(_p(Wp), float(np.float32(gamma)), N, K, _p(x), M, _p(res),
                          _p(y), _p(acc), _p(xq), _p(s), _p(xs))
    if rc != 0:
        raise MemoryError("oracle forward failed")
    return dict(y=y, acc=acc, xq=xq, s=s, xsum=xs)


def forward_ex(Wp: np.ndarray, gammas, seg_rows, x_bf16: np.ndarray, rmsnorm=False, residual=None):
    """Projections of one input against row-stacked weight matrices (segment i:
    seg_rows[i] rows, gamma gammas[i]), optionally after a unit-weight RMSNorm of
    the input. Returns dict(y, acc); y as bf16 bits [M, N]."""
    Wp = _c(Wp, np.uint8)
    x = _c(x_bf16, np.uint16)
    g = _c(np.asarray(gammas, np.float32), np.float32)
    rows = _c(np.asarray(seg_rows, np.int64), np.int64)
    N = int(rows.sum())
    M, K = x.shape
    assert Wp.shape == (N, K // 4) and g.size == rows.size
    res = None if residual is None else _c(residual, np.uint16)
    y = np.empty((M, N), np.uint16)
    acc = np.empty((M, N), np.int32)
    rc = _l().orc_forward_ex(_p(Wp), _p(g), _p(rows), rows.size, K, _p(x), M, int(bool(rmsnorm)), _p(res),
                             _p(y), _p(acc))
    if rc != 0:
        raise MemoryError("oracle forward_ex failed")
    return dict(y=y, acc=acc)


def pack_weights_rowwise(W: np.ndarray):
    """Per-row absmean variant: W [N, K] (fp32, or bf16 bits) -> (Wp uint8 [N, K/4], gammas fp32 [N])."""
    if W.dtype == np.uint16:
        W = bf16_to_f32(W)
    W = _c(W, np.float32)
    N, K = W.shape
    Wp = np.empty((N, K // 4), np.uint8)
    g = np.empty(N, np.float32)
    if _l().orc_pack_weights_rowwise(_p(W), N, K, _p(Wp), _p(g)) != 0:
        raise MemoryError("oracle pack_weights_rowwise failed")
    return Wp, g


def forward_rowwise(Wp: np.ndarray, gammas: np.ndarray, x_bf16: np.ndarray, residual=None):
    """Forward with one gamma per output row. Returns dict(y, acc); y as bf16 bits."""
    Wp = _c(Wp, np.uint8)
    x = _c(x_bf16, np.uint16)
    g = _c(np.asarray(gammas, np.float32), np.float32)
    N = Wp.shape[0]
    M, K = x.shape
    assert Wp.shape[1] * 4 == K and g.size == N
    res = None if residual is None else _c(residual, np.uint16)
    y = np.empty((M, N), np.uint16)
    acc = np.empty((M, N), np.int32)
    if _l().orc_forward_rowwise(_p(Wp), _p(g), N, K, _p(x), M, _p(res), _p(y), _p(acc)) != 0:
        raise MemoryError("oracle forward_rowwise failed")
    return dict(y=y, acc=acc)


def subln_rms(h: np.ndarray):
    h = _c(h, np.float32)
    hn = np.empty_like(h)
    r = _l().orc_subln_rms(_p(h), h.size, _p(hn))
    return np.float32(r), hn


def relu2_gate(g, u) -> np.float32:
    return np.float32(_l().orc_relu2_gate(float(np.float32(g)), float(np.float32(u))))


def ffn_layer(Wg, gg, Wu, gu, Wd, gd, x_bf16, residual=None):
    """One FFN sub-layer; returns dict(y, h, q2, s2, r, accd); y as bf16 bits."""
    Wg = _c(Wg, np.uint8)
    Wu = _c(Wu, np.uint8)
    Wd = _c(Wd, np.uint8)
    x = _c(x_bf16, np.uint16)
    M, d = x.shape
    f = Wg.shape[0]
    assert Wg.shape == (f, d // 4) and Wu.shape == (f, d // 4) and Wd.shape == (d, f // 4)
    res = None if residual is None else _c(residual, np.uint16)
    y = np.empty((M, d), np.uint16)
    h = np.empty((M, f), np.float32)
    q2 = np.empty((M, f), np.int8)
    s2 = np.empty(M, np.float32)
    r = np.empty(M, np.float32)
    accd = np.empty((M, d), np.int32)
    rc = _l().orc_ffn_layer(_p(Wg), float(np.float32(gg)), _p(Wu), float(np.float32(gu)),
                            _p(Wd), float(np.float32(gd)), d, f, _p(x), M, _p(res), _p(y),
                            _p(h), _p(q2), _p(s2), _p(r), _p(accd))
    if rc != 0:
        raise MemoryError("oracle ffn_layer failed")
    return dict(y=y, h=h, q2=q2, s2=s2, r=r, accd=accd)


# --------------------------------------------------------------------------- tensor-parallel pieces

def absmean_sum(W: np.ndarray) -> float:
    """fp64 sum of |W| of one shard (fp32, or bf16 bits)."""
    if W.dtype == np.uint16:
        W = bf16_to_f32(W)
    W = _c(W, np.float32)
    return float(_l().orc_absmean_sum(_p(W), W.size))


def pack_weights_global(W: np.ndarray, total_sum: float, total_count: int):
    """Pack one shard with gamma = fp32(total_sum / total_count) of the whole tensor."""
    if W.dtype == np.uint16:
        W = bf16_to_f32(W)
    W = _c(W, np.float32)
    N, K = W.shape
    Wp = np.empty((N, K // 4), np.uint8)
    g = np.zeros(1, np.float32)
    if _l().orc_pack_weights_global(_p(W), N, K, float(total_sum), int(total_count), _p(Wp), _p(g)) != 0:
        raise MemoryError("oracle pack_weights_global failed")
    return Wp, np.float32(g[0])


def ffn_tp_up(Wg, gg, Wu, gu, x_bf16):
    """Rank-local gate/up: returns (h [M, fl] fp32, ss [M] fp64, hmax [M] fp32)."""
    Wg = _c(Wg, np.uint8)
    Wu = _c(Wu, np.uint8)
    x = _c(x_bf16, np.uint16)
    M, d = x.shape
    fl = Wg.shape[0]
    assert Wg.shape == (fl, d // 4) and Wu.shape == (fl, d // 4)
    h = np.empty((M, fl), np.float32)
    ss = np.empty(M, np.float64)
    hmax = np.empty(M, np.float32)
    if _l().orc_ffn_tp_up(_p(Wg), float(np.float32(gg)), _p(Wu), float(np.float32(gu)), d, fl, _p(x), M, _p(h),
                          _p(ss), _p(hmax)) != 0:
        raise MemoryError("oracle ffn_tp_up failed")
    return h, ss, hmax


def ffn_tp_down(Wd, h, ss_all, hmax_all, f_total: int):
    """Rank-local requantisation with the global statistics and the partial down
    projection: returns (acc [M, d] int32, s2 [M] fp32)."""
    Wd = _c(Wd, np.uint8)
    h = _c(h, np.float32)
    ss_all = _c(ss_all, np.float64)
    hmax_all = _c(hmax_all, np.float32)
    M, fl = h.shape
    d = Wd.shape[0]
    assert Wd.shape == (d, fl // 4)
    acc = np.empty((M, d), np.int32)
    s2 = np.empty(M, np.float32)
    if _l().orc_ffn_tp_down(_p(Wd), d, fl, int(f_total), _p(h), M, _p(ss_all), _p(hmax_all), _p(acc),
                            _p(s2)) != 0:
        raise MemoryError("oracle ffn_tp_down failed")
    return acc, s2

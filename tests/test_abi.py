"""The C ABI library: it loads, exports every declared symbol, and rejects bad
arguments on the host before touching a GPU (CPU only; no compute calls)."""
import ctypes
import os
import re

import pytest
import torch

import bitlinear_w1_a8_02_b200 as bl
from bitlinear_w1_a8_02_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")

# bl_status codes, as include/bitlinear.h numbers them
OK, NULL, SHAPE, ALIGN, DTYPE, WS, UNSUP = 0, 1, 2, 3, 4, 5, 6


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 8
    L = bl.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(binding.SIGNATURES)


def test_library_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {bl.LIB_PATH}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    ours = {n for n in exported if n.startswith("bitlinear_")}
    assert ours == set(declared_functions())


def test_status_strings():
    L = bl.lib()
    for code, name in binding.STATUS_NAMES.items():
        s = L.bitlinear_status_string(code).decode()
        assert s.startswith(name), (code, s)
    assert L.bitlinear_status_string(1234).decode() == "unknown bl_status"


def test_workspace_sizes():
    L = bl.lib()
    f = L.bitlinear_workspace_bytes
    assert f(bl.BL_OP_FORWARD, 1, 2560, 2560) >= 2560 + 8
    assert f(bl.BL_OP_FORWARD, 16, 6912, 2560) >= 16 * 2560
    assert f(bl.BL_OP_FFN, 512, 6912, 2560) >= 512 * 6912 * 9
    assert f(bl.BL_OP_PACK, 0, 512, 256) >= 8
    assert f(bl.BL_OP_VALIDATE, 0, 0, 0) == 256
    assert f(99, 1, 1, 4) == 0
    assert f(bl.BL_OP_FORWARD, -1, 1, 4) == 0
    for op in (bl.BL_OP_FORWARD, bl.BL_OP_FFN):
        assert f(op, 1, 2560, 2560) % 256 == 0
    # tensor-core shapes that take the stream-K split carry its scratch (two
    # 128 x 256 int32 slots per SM, sized for 148 SMs without asking a device);
    # shapes that keep the data-parallel split and the M <= 16 paths do not
    sk = 2 * 148 * 128 * 256 * 4
    assert f(bl.BL_OP_FORWARD, 512, 2560, 6912) >= 512 * 6912 + sk   # 40 tiles of 54 k-blocks
    assert f(bl.BL_OP_FFN, 512, 6912, 2560) >= sk                     # its down projection
    assert f(bl.BL_OP_FORWARD, 17, 2560, 2560) < sk                   # 20 k-blocks: data-parallel
    assert f(bl.BL_OP_FORWARD, 4096, 6912, 2560) < sk                 # 864 tiles fill the waves
    assert f(bl.BL_OP_FORWARD, 16, 2560, 2560) < sk


# Fake, never-dereferenced addresses: every call below must fail host-side
# validation before any CUDA call.
A = 0x10000  # 64 KiB aligned
P = ctypes.c_void_p


def test_host_validation_forward():
    L = bl.lib()
    F = L.bitlinear_forward
    ws_need = L.bitlinear_workspace_bytes(bl.BL_OP_FORWARD, 1, 512, 256)
    args = dict(Wp=A, g=A, N=512, K=256, x=A, M=1, res=None, y=A, acc=None, ws=A, wsb=ws_need)

    def call(**kw):
        a = dict(args, **kw)
        return F(P(a["Wp"]), P(a["g"]), a["N"], a["K"], P(a["x"]), a["M"], P(a["res"]), P(a["y"]),
                 P(a["acc"]), P(a["ws"]), a["wsb"], None)

    assert call(K=258) == SHAPE
    assert call(K=0) == SHAPE
    assert call(M=-1) == SHAPE
    assert call(N=-3) == SHAPE
    assert call(M=70000) == SHAPE
    assert call(K=1 << 20) == SHAPE
    assert call(M=0) == OK          # empty: nothing to do
    assert call(N=0) == OK
    assert call(Wp=None) == NULL
    assert call(x=None) == NULL
    assert call(y=None) == NULL
    assert call(g=None) == NULL
    assert call(g=A + 2) == ALIGN
    assert call(y=A + 1) == ALIGN
    assert call(acc=A + 2) == ALIGN
    assert call(ws=A + 16) == ALIGN
    assert call(ws=None) == NULL
    assert call(wsb=ws_need - 1) == WS


def test_host_validation_pack_quant_ffn_validate():
    L = bl.lib()
    need = L.bitlinear_workspace_bytes(bl.BL_OP_PACK, 0, 8, 16)
    pk = L.bitlinear_pack_weights
    assert pk(P(A), 7, 8, 16, P(A), P(A), P(A), need, None) == DTYPE
    assert pk(P(A), bl.BL_BF16, 0, 16, P(A), P(A), P(A), need, None) == SHAPE
    assert pk(P(A), bl.BL_BF16, 8, 18, P(A), P(A), P(A), need, None) == SHAPE
    assert pk(None, bl.BL_BF16, 8, 16, P(A), P(A), P(A), need, None) == NULL
    assert pk(P(A + 8), bl.BL_BF16, 8, 16, P(A), P(A), P(A), need, None) == ALIGN
    assert pk(P(A), bl.BL_BF16, 8, 16, P(A), P(A), P(A), need - 1, None) == WS

    q = L.bitlinear_quant_act
    assert q(P(A), 2, 6, P(A), P(A), None, None) == SHAPE
    assert q(P(A), 0, 8, None, None, None, None) == OK
    assert q(None, 2, 8, P(A), P(A), None, None) == NULL
    assert q(P(A), 2, 8, P(A), P(A + 1), None, None) == ALIGN

    ffn = L.bitlinear_ffn
    need = L.bitlinear_workspace_bytes(bl.BL_OP_FFN, 1, 32, 16)
    base = [P(A)] * 6
    assert ffn(*base, 16, 30, P(A), 1, None, P(A), P(A), need, None) == SHAPE
    assert ffn(*base, 16, 32, P(A), 0, None, P(A), P(A), need, None) == OK
    assert ffn(*base[:5], None, 16, 32, P(A), 1, None, P(A), P(A), need, None) == NULL
    assert ffn(*base, 16, 32, P(A), 1, None, P(A), P(A), need - 1, None) == WS

    v = L.bitlinear_validate_packed
    cnt = ctypes.c_int64(-1)
    assert v(P(A), 4, 6, ctypes.byref(cnt), P(A), 256, None) == SHAPE
    assert v(P(A), 0, 16, ctypes.byref(cnt), P(A), 256, None) == OK and cnt.value == 0
    assert v(None, 4, 16, None, P(A), 256, None) == NULL


def test_host_validation_forward_ex():
    L = bl.lib()
    F = L.bitlinear_forward_ex
    need = L.bitlinear_workspace_bytes(bl.BL_OP_FORWARD, 1, 96, 256)

    def call(rows, nseg=None, K=256, M=1, norm=0, g=A, ws=A, wsb=need):
        arr = None if rows is None else (ctypes.c_int64 * max(1, len(rows)))(*rows)
        n = len(rows) if nseg is None else nseg
        return F(P(A), P(g), arr, n, K, P(A), M, norm, None, P(A), None, P(ws), wsb, None)

    assert call([48, 16, 32], nseg=0) == SHAPE
    assert call([48, 16, 32, 8, 8], nseg=5) == SHAPE
    assert call([48, 0, 32]) == SHAPE
    assert call([48, 16, 32], norm=2) == SHAPE
    assert call([48, 16, 32], K=258) == SHAPE
    assert call(None, nseg=3) == NULL
    assert call([48, 16, 32], M=0) == OK
    assert call([48, 16, 32], g=None) == NULL
    assert call([48, 16, 32], g=A + 2) == ALIGN
    assert call([48, 16, 32], wsb=need - 1) == WS


def test_host_validation_rowwise():
    L = bl.lib()
    pk = L.bitlinear_pack_weights_rowwise
    assert pk(P(A), 7, 8, 16, P(A), P(A), None) == DTYPE
    assert pk(P(A), bl.BL_BF16, 8, 18, P(A), P(A), None) == SHAPE
    assert pk(P(A), bl.BL_BF16, 0, 16, P(A), P(A), None) == SHAPE
    assert pk(P(A), bl.BL_BF16, 8, 16, P(A), None, None) == NULL
    assert pk(P(A + 8), bl.BL_BF16, 8, 16, P(A), P(A), None) == ALIGN
    F = L.bitlinear_forward_rowwise
    need = L.bitlinear_workspace_bytes(bl.BL_OP_FORWARD, 1, 512, 256)
    assert F(P(A), P(A), 512, 258, P(A), 1, None, P(A), None, P(A), need, None) == SHAPE
    assert F(P(A), P(A), 512, 256, P(A), 0, None, P(A), None, P(A), need, None) == OK
    assert F(P(A), None, 512, 256, P(A), 1, None, P(A), None, P(A), need, None) == NULL
    assert F(P(A), P(A + 2), 512, 256, P(A), 1, None, P(A), None, P(A), need, None) == ALIGN
    assert F(P(A), P(A), 512, 256, P(A), 1, None, P(A), None, P(A), need - 1, None) == WS


def test_host_validation_tensor_parallel():
    """The five tensor-parallel calls reject bad dtypes, shapes, pointers,
    alignments and workspaces on the host, and treat M = 0 as a no-op."""
    L = bl.lib()
    need = L.bitlinear_workspace_bytes(bl.BL_OP_PACK, 0, 8, 16)
    asum = L.bitlinear_absmean_sum
    assert asum(P(A), 7, 8, 16, P(A), P(A), need, None) == DTYPE
    assert asum(P(A), bl.BL_BF16, 0, 16, P(A), P(A), need, None) == SHAPE
    assert asum(P(A), bl.BL_BF16, 8, 18, P(A), P(A), need, None) == SHAPE
    assert asum(P(A), bl.BL_BF16, 8, 16, None, P(A), need, None) == NULL
    assert asum(P(A), bl.BL_BF16, 8, 16, P(A + 4), P(A), need, None) == ALIGN
    assert asum(P(A), bl.BL_BF16, 8, 16, P(A), P(A), need - 1, None) == WS

    glob = L.bitlinear_pack_weights_global
    assert glob(P(A), 7, 8, 16, P(A), 256, P(A), P(A), None) == DTYPE
    assert glob(P(A), bl.BL_BF16, 8, 16, P(A), 127, P(A), P(A), None) == SHAPE  # count below N * K
    assert glob(P(A), bl.BL_BF16, 8, 16, None, 256, P(A), P(A), None) == NULL
    assert glob(P(A), bl.BL_BF16, 8, 16, P(A + 4), 256, P(A), P(A), None) == ALIGN

    up = L.bitlinear_ffn_tp_up
    need = L.bitlinear_workspace_bytes(bl.BL_OP_FFN_TP_UP, 2, 256, 64)
    w4 = [P(A)] * 4

    def call_up(d=64, fl=256, M=2, h=A, ss=A, ws=A, wsb=need):
        return up(*w4, d, fl, P(A), M, P(h), P(ss), P(A), P(ws), wsb, None)

    assert call_up(d=66) == SHAPE
    assert call_up(fl=2) == SHAPE
    assert call_up(M=-1) == SHAPE
    assert call_up(M=0) == OK
    assert call_up(h=None) == NULL
    assert call_up(ss=A + 4) == ALIGN
    assert call_up(ws=A + 16) == ALIGN
    assert call_up(wsb=need - 1) == WS

    down = L.bitlinear_ffn_tp_down
    need = L.bitlinear_workspace_bytes(bl.BL_OP_FFN_TP_DOWN, 2, 64, 256)

    def call_down(d=64, fl=256, f_total=512, M=2, ss=A, acc=A, wsb=need):
        return down(P(A), d, fl, f_total, P(A), M, P(ss), P(A), P(acc), P(A), P(A), wsb, None)

    assert call_down(f_total=200) == SHAPE   # the whole width below the rank's share
    assert call_down(fl=258) == SHAPE
    assert call_down(d=0) == SHAPE
    assert call_down(M=0) == OK
    assert call_down(acc=None) == NULL
    assert call_down(ss=A + 4) == ALIGN
    assert call_down(wsb=need - 1) == WS

    fin = L.bitlinear_ffn_tp_finish
    assert fin(P(A), P(A), P(A), None, P(A), -1, 64, None) == SHAPE
    assert fin(P(A), P(A), P(A), None, P(A), 0, 64, None) == OK
    assert fin(P(A), None, P(A), None, P(A), 2, 64, None) == NULL
    assert fin(P(A), P(A), P(A), P(A + 1), P(A), 2, 64, None) == ALIGN


def test_host_validation_noalloc():
    """The allocation-free forward checks its arguments like bitlinear_forward, and
    refuses sizes whose codes and per-token words would not fit its fixed 1 MiB
    scratch, before touching a device."""
    F = bl.lib().bitlinear_forward_noalloc

    def call(N=512, K=256, M=1, g=A, x=A, y=A, res=None, acc=None):
        return F(P(A), P(g), N, K, P(x), M, P(res), P(y), P(acc), None)

    assert call(K=258) == SHAPE
    assert call(M=-1) == SHAPE
    assert call(N=-1) == SHAPE
    assert call(M=0) == OK
    assert call(N=0) == OK
    assert call(x=None) == NULL
    assert call(g=None) == NULL
    assert call(g=A + 2) == ALIGN
    assert call(y=A + 1) == ALIGN
    assert call(res=A + 1) == ALIGN
    assert call(acc=A + 2) == ALIGN
    assert call(M=64, K=32768) == WS      # 2 MiB of codes


def test_host_validation_selftest():
    L = bl.lib()
    assert L.bitlinear_selftest_timeout(0, None) == SHAPE
    assert L.bitlinear_selftest_timeout(3_000_000, None) == SHAPE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device answer")
def test_valid_call_without_device_is_unsupported():
    L = bl.lib()
    need = L.bitlinear_workspace_bytes(bl.BL_OP_FORWARD, 1, 512, 256)
    st = L.bitlinear_forward(P(A), P(A), 512, 256, P(A), 1, None, P(A), None, P(A), need, None)
    assert st == UNSUP
    st = L.bitlinear_forward_noalloc(P(A), P(A), 512, 256, P(A), 1, None, P(A), None, None)
    assert st == UNSUP
    assert L.bitlinear_get_device_error(None) == UNSUP


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        binding.lib()

"""The allocation-free forward, called through the C ABI.

bitlinear_forward_noalloc serves callers that cannot allocate device memory
where they run a layer (an engine that reserved all of it at start-up, or a
loop where an allocation would synchronise the device) and so cannot hand over
a workspace either. It keeps its scratch in a fixed array in the library's own
device memory. These tests check that two calls in a row give what
bitlinear_forward gives (bit for bit, and within the tolerance the other parity
tests use) and what the CPU oracle gives, on the streamed GEMV, the generic
kernel (K % 256 != 0, and an x that is only 2-byte aligned) and more than 16
tokens, and that sizes beyond the array are refused. The file is collected last
and passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import bitlinear_w1_a8_02_b200 as bl
import oracle
from bitlinear_w1_a8_02_b200 import synth
from gpu_util import assert_bf16_close, assert_bf16_exact, bits, np_

pytestmark = pytest.mark.gpu

BL_ERR_WORKSPACE = 5
SCRATCH_BYTES = 1 << 20


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def noalloc(Wp, gamma, x, residual=None):
    N, KB = Wp.shape
    M, K = x.shape
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=x.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream(x.device).cuda_stream)
    st = bl.lib().bitlinear_forward_noalloc(_p(Wp), _p(gamma), N, K, _p(x), M, _p(residual),
                                            _p(y), _p(acc), stream)
    return st, y, acc


def _unaligned(x):
    """The same values as x, starting 2 bytes past a 16-byte boundary."""
    M, K = x.shape
    buf = torch.empty(M * K + 8, dtype=torch.bfloat16, device=x.device)
    v = buf[1:1 + M * K].view(M, K)
    v.copy_(x)
    return v


# (K, N, M, residual, unaligned x): the streamed GEMV at M = 1 and 16, the generic
# kernel for K % 256 != 0 and for an x that is only 2-byte aligned, and M > 16.
CASES = [(2560, 6912, 1, True, False), (6912, 2560, 16, False, False), (2564, 640, 3, True, False),
         (2560, 640, 5, False, True), (2560, 2560, 64, True, False)]


def test_noalloc_matches_forward_and_oracle_on_calls_in_a_row(cuda_device):
    prepared = []
    for i, (K, N, M, use_res, unaligned) in enumerate(CASES):
        W = synth.weights(N, K, synth.SIGMA_2B, seed=500 + i)
        Wp, gamma = bl.pack_weights(W.to(cuda_device))
        x_cpu = synth.activations(M, K, seed=600 + i, outliers=True)
        x = x_cpu.to(cuda_device)
        if unaligned:
            x = _unaligned(x)
            assert x.data_ptr() % 16 == 2
        res_cpu = synth.activations(M, N, seed=700 + i, outliers=False) if use_res else None
        res = None if res_cpu is None else res_cpu.to(cuda_device)
        y_ref, acc_ref = bl.forward(Wp, gamma, x, residual=res, want_acc=True)
        prepared.append((Wp, gamma, x, x_cpu, res, res_cpu, y_ref, acc_ref))
    torch.cuda.synchronize()
    # the calls back to back on one stream; each overwrites the previous one's scratch
    outs = [noalloc(Wp, gamma, x, res) for (Wp, gamma, x, _, res, _, _, _) in prepared]
    torch.cuda.synchronize()
    for (st, y, acc), (Wp, gamma, _, x_cpu, _, res_cpu, y_ref, acc_ref) in zip(outs, prepared):
        assert st == 0
        assert np.array_equal(np_(acc), np_(acc_ref))
        assert_bf16_close(bits(y), bits(y_ref))
        assert_bf16_exact(bits(y), bits(y_ref))
        ref = oracle.forward(np_(Wp), np_(gamma)[0], bits(x_cpu),
                             residual=None if res_cpu is None else bits(res_cpu))
        assert np.array_equal(np_(acc), ref["acc"])
        assert_bf16_exact(bits(y), ref["y"])
    assert bl.get_device_error() == 0


def test_noalloc_refuses_sizes_beyond_its_scratch(cuda_device):
    K, N = 2560, 640
    Wp, gamma = bl.pack_weights(synth.weights(N, K, synth.SIGMA_2B, seed=9, device=cuda_device))
    M = SCRATCH_BYTES // K + 1
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=cuda_device)
    st, _, _ = noalloc(Wp, gamma, x)
    assert st == BL_ERR_WORKSPACE

"""The allocation-free forward, called through the C ABI.

bitlinear_forward_noalloc serves callers that cannot allocate device memory
where they run a layer (an engine that reserved all of it at start-up, or a
loop where an allocation would synchronise the device) and so cannot hand over
a workspace either. It keeps its scratch in a fixed array in the library's own
device memory. This test checks that two calls in a row give what
bitlinear_forward gives, within the tolerance the other parity tests use, and
that sizes beyond the array are refused. It lives in its own file, collected
last, and passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import bitlinear_w1_a8_02_b200 as bl
from bitlinear_w1_a8_02_b200 import synth
from gpu_util import assert_bf16_close, bits, np_

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


def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_device):
    cases = [(2560, 6912, 1, True), (6912, 2560, 16, False)]  # (K, N, M, residual)
    prepared = []
    for i, (K, N, M, use_res) in enumerate(cases):
        W = synth.weights(N, K, synth.SIGMA_2B, seed=500 + i, device=cuda_device)
        Wp, gamma = bl.pack_weights(W)
        x = synth.activations(M, K, seed=600 + i, outliers=True, device=cuda_device)
        res = synth.activations(M, N, seed=700 + i, outliers=False, device=cuda_device) if use_res else None
        y_ref, acc_ref = bl.forward(Wp, gamma, x, residual=res, want_acc=True)
        prepared.append((Wp, gamma, x, res, y_ref, acc_ref))
    torch.cuda.synchronize()
    # two calls back to back on one stream; the second overwrites the first's scratch
    outs = [noalloc(Wp, gamma, x, res) for (Wp, gamma, x, res, _, _) in prepared]
    torch.cuda.synchronize()
    for (st, y, acc), (_, _, _, _, y_ref, acc_ref) in zip(outs, prepared):
        assert st == 0
        assert np.array_equal(np_(acc), np_(acc_ref))
        assert_bf16_close(bits(y), bits(y_ref))
    assert bl.get_device_error() == 0


def test_noalloc_refuses_sizes_beyond_its_scratch(cuda_device):
    K, N = 2560, 640
    Wp, gamma = bl.pack_weights(synth.weights(N, K, synth.SIGMA_2B, seed=9, device=cuda_device))
    M = SCRATCH_BYTES // K + 1
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=cuda_device)
    st, _, _ = noalloc(Wp, gamma, x)
    assert st == BL_ERR_WORKSPACE

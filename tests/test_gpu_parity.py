"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integers (packed bytes, gamma bits, activation codes, scales, accumulators) must
match bit for bit; bf16 outputs must meet the 2^-8 relative bar and, because
every fp32 step is a unique IEEE result in both implementations, also match bit
for bit. Full-size workloads compare sampled rows and tokens, each computed by
the oracle on the same inputs.
"""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_02_b200 as bl
import oracle
from bitlinear_w1_a8_02_b200 import synth
from gpu_util import assert_bf16_close, assert_bf16_exact, bits, np_, sample_indices

pytestmark = pytest.mark.gpu


def make_weights(N, K, sigma, seed, dtype="bf16"):
    return synth.weights(N, K, sigma, seed, dtype=dtype)


def pack_both(W_cpu: torch.Tensor, dev):
    """Pack on the GPU and in the oracle; assert identical bytes and gamma."""
    Wp, gamma = bl.pack_weights(W_cpu.to(dev))
    if W_cpu.dtype == torch.bfloat16:
        Wp_ref, g_ref = oracle.pack_weights(bits(W_cpu))
    else:
        Wp_ref, g_ref = oracle.pack_weights(np_(W_cpu))
    assert np_(gamma)[0].view(np.uint32) == np.float32(g_ref).view(np.uint32), "gamma bits"
    assert np.array_equal(np_(Wp), Wp_ref), "packed bytes"
    return Wp, gamma, Wp_ref, g_ref


def check_forward_full(Wp, gamma, Wp_ref, g_ref, x_cpu, dev, residual=None):
    y, acc = bl.forward(Wp, gamma, x_cpu.to(dev), residual=None if residual is None else residual.to(dev),
                        want_acc=True)
    ref = oracle.forward(Wp_ref, g_ref, bits(x_cpu), residual=None if residual is None else bits(residual))
    assert np.array_equal(np_(acc), ref["acc"]), "int32 accumulators"
    assert_bf16_close(bits(y), ref["y"])
    assert_bf16_exact(bits(y), ref["y"])


def check_forward_sampled(Wp, gamma, Wp_ref, g_ref, x_cpu, dev, rows, toks):
    y, acc = bl.forward(Wp, gamma, x_cpu.to(dev), want_acc=True)
    ref = oracle.forward(Wp_ref[rows], g_ref, bits(x_cpu[toks]))
    got_acc = np_(acc)[np.ix_(toks, rows)]
    assert np.array_equal(got_acc, ref["acc"]), "int32 accumulators (sampled)"
    got_y = bits(y)[np.ix_(toks, rows)]
    assert_bf16_close(got_y, ref["y"])
    assert_bf16_exact(got_y, ref["y"])


# ----------------------------------------------------------------------------- packing

@pytest.mark.parametrize("N,K,dtype", [(512, 256, "fp32"), (2560, 2560, "bf16"), (640, 2560, "bf16"),
                                       (6912, 2560, "bf16"), (2560, 6912, "bf16"), (136, 196, "bf16"),
                                       (1, 4, "fp32"), (3, 12, "bf16")])
def test_pack_parity(cuda_device, N, K, dtype):
    pack_both(make_weights(N, K, 0.02, seed=N + K, dtype=dtype), cuda_device)


def test_pack_parity_100b_shape(cuda_device):
    W = make_weights(8192, 28672, synth.SIGMA_100B, seed=77)
    Wp, gamma, Wp_ref, _ = pack_both(W, cuda_device)
    assert bl.validate_packed(Wp) == 0


def test_validate_packed_counts_bad_codes(cuda_device):
    Wp, _ = bl.pack_weights(make_weights(64, 256, 0.02, seed=3).to(cuda_device))
    assert bl.validate_packed(Wp) == 0
    Wp[3, 5] = 0xFF   # four invalid codes
    Wp[10, 0] = 0x57  # one invalid code (field 0 = 3)
    assert bl.validate_packed(Wp) == 5


# ----------------------------------------------------------------------------- act-quant

@pytest.mark.parametrize("M,K", [(1, 256), (7, 2560), (33, 6912), (4, 260), (2, 4), (5, 28672)])
def test_quant_act_parity(cuda_device, M, K):
    x = synth.activations(M, K, seed=M * 7 + K, outliers=True)
    if M > 2:
        x[1] = 0
        x[2] = x[2] * 1e-7
    xq, s, xs = bl.quant_act(x.to(cuda_device))
    rq, rs, rxs = oracle.quant_act(bits(x))
    assert np.array_equal(np_(xq), rq)
    assert np.array_equal(np_(s).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(np_(xs), rxs)


def test_quant_act_empty(cuda_device):
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=cuda_device)
    xq, s, xs = bl.quant_act(x)
    assert xq.shape == (0, 256)


# ----------------------------------------------------------------------------- forward

def test_forward_single_fp32_weights(cuda_device):
    """The small case: M=1, K=256, N=512, fp32 W ~ N(0, 0.02^2), x ~ N(0, 1), seed 0."""
    W = make_weights(512, 256, 0.02, seed=0, dtype="fp32")
    x = synth.activations(1, 256, seed=0, outliers=False)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)


@pytest.mark.parametrize("K,N", [(2560, 2560), (2560, 640), (2560, 6912), (6912, 2560)])
def test_forward_decode_2b(cuda_device, K, N):
    W = make_weights(N, K, 0.02, seed=1000 + K + N)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(1, K, seed=1, outliers=True)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)


@pytest.mark.parametrize("M", [2, 4, 8, 9, 16])
@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560)])
def test_forward_batched_decode(cuda_device, K, N, M):
    W = make_weights(N, K, 0.02, seed=2000 + K + N)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=M, outliers=True)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)


@pytest.mark.parametrize("K,N,M", [(8192, 28672, 4), (6912, 2560, 4), (6912, 2560, 3), (2560, 2560, 3)])
def test_forward_few_tokens_quantiser_routes(cuda_device, K, N, M):
    """2 to 4 tokens take one of three quantisation routes: the in-kernel
    quantiser that loads every token's group at once (K <= 4096), the per-token
    in-kernel loop (K > 4096, or four tokens on a large grid: 8192 -> 28672 has
    1792 16-row tiles), or the separate act-quant kernel (four tokens with
    K > 4096 on a grid of at most two tiles per SM: 6912 -> 2560). All must give
    the oracle's bits; the large shape is checked on sampled rows."""
    W = make_weights(N, K, synth.SIGMA_100B if K * N > 10**8 else 0.02, seed=7000 + K + M)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=7100 + M, outliers=True)
    if K * N > 10**8:
        rows = sample_indices(N, 256, seed=M + 71)
        check_forward_sampled(Wp, gamma, Wp_ref, g_ref, x, cuda_device, rows, np.arange(M))
    else:
        check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)


@pytest.mark.parametrize("M", [17, 512, 2048, 4096])
@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560)])
def test_forward_prefill_sampled(cuda_device, K, N, M):
    W = make_weights(N, K, 0.02, seed=3000 + K + N)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=M + 5, outliers=True)
    rows = sample_indices(N, 96, seed=M)
    toks = sample_indices(M, 12, seed=M + 1)
    check_forward_sampled(Wp, gamma, Wp_ref, g_ref, x, cuda_device, rows, toks)


@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560)])
def test_forward_prefill_full_output(cuda_device, K, N):
    """Every output of a 512-token prefill at the 2B FFN shapes (the tensor-core
    GEMM, stream-K split for 6912 -> 2560) against the oracle."""
    M = 512
    W = make_weights(N, K, 0.02, seed=3100 + K + N)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=3200 + M, outliers=True)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)


@pytest.mark.parametrize("M", [1, 16, 2048])
@pytest.mark.parametrize("K,N", [(8192, 28672), (28672, 8192)])
def test_forward_100b_sampled(cuda_device, K, N, M):
    W = make_weights(N, K, synth.SIGMA_100B, seed=4000 + K % 1000)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=M + 9, outliers=True)
    rows = sample_indices(N, 64, seed=M + 2)
    toks = sample_indices(M, 8, seed=M + 3)
    check_forward_sampled(Wp, gamma, Wp_ref, g_ref, x, cuda_device, rows, toks)


@pytest.mark.parametrize("M,N,K", [(17, 136, 192), (3, 17, 256), (1, 1, 4), (5, 33, 260),
                                   (16, 130, 512), (20, 100, 1024)])
def test_forward_ragged_shapes(cuda_device, M, N, K):
    W = make_weights(N, K, 0.02, seed=M + N + K)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=K, outliers=True)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)


@pytest.mark.parametrize("M,N,K", [(129, 257, 64), (300, 512, 320), (33, 1000, 2560),
                                   (4096, 256, 128), (17, 8, 64), (512, 2400, 128), (64, 1000, 192)])
def test_forward_tensor_core_tails(cuda_device, M, N, K):
    """M > 16 runs the tcgen05 GEMM: token, row and k-block tails, N not a
    multiple of the weight-row tile, K not a multiple of the 128-code k-block.
    The last two shapes pick the 128- and 64-row tiles."""
    W = make_weights(N, K, 0.02, seed=M + 3 * N + K)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=N, outliers=True)
    res = synth.activations(M, N, seed=K, outliers=False)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device, residual=res)


@pytest.mark.parametrize("M,N,K", [(200, 600, 4096), (300, 2560, 4160)])
def test_forward_stream_k_split_tiles(cuda_device, M, N, K):
    """Few tiles and at least 32 k-blocks: the GEMM splits tiles across CTAs
    (stream-K) and a second kernel sums the int32 pieces. Ragged tokens, rows and
    last k-block; with and without the residual."""
    W = make_weights(N, K, 0.02, seed=M + N + 7 * K)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=M + 1, outliers=True)
    res = synth.activations(M, N, seed=N + 1, outliers=False)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device, residual=res)


def stacked(shapes_rows, K, seed, dev):
    """Pack each matrix on the GPU and in the oracle; stack rows and gammas."""
    parts = [pack_both(make_weights(n, K, synth.SIGMA_2B, seed + i), dev) for i, n in enumerate(shapes_rows)]
    Wp = torch.cat([p[0] for p in parts])
    gam = torch.cat([p[1].reshape(1) for p in parts])
    Wp_ref = np.concatenate([p[2] for p in parts])
    g_ref = [p[3] for p in parts]
    return Wp, gam, Wp_ref, g_ref


@pytest.mark.parametrize("M", [1, 3, 9, 40, 300])
@pytest.mark.parametrize("norm", [False, True])
def test_forward_ex_qkv(cuda_device, M, norm):
    """The attention's query/key/value projections (2560 -> 2560 / 640 / 640) of
    one input in one call, with and without the block's pre-norm: single-token
    dp4a GEMV, fused multi-token GEMV, act-quant + GEMV, and the tensor-core GEMM."""
    K, rows = 2560, [2560, 640, 640]
    Wp, gam, Wp_ref, g_ref = stacked(rows, K, 80, cuda_device)
    x = synth.activations(M, K, seed=81 + M, outliers=True)
    y, acc = bl.forward_ex(Wp, gam, rows, x.to(cuda_device), rmsnorm=norm, want_acc=True)
    ref = oracle.forward_ex(Wp_ref, g_ref, rows, bits(x), rmsnorm=norm)
    assert np.array_equal(np_(acc), ref["acc"]), "int32 accumulators"
    assert_bf16_close(bits(y), ref["y"])
    assert_bf16_exact(bits(y), ref["y"])


@pytest.mark.parametrize("M", [1, 4, 17])
def test_forward_ex_output_projection_with_subln(cuda_device, M):
    """The attention output projection (2560 -> 2560): subln RMSNorm of the
    attention output, quantisation, projection, residual add."""
    K, rows = 2560, [2560]
    Wp, gam, Wp_ref, g_ref = stacked(rows, K, 90, cuda_device)
    x = synth.activations(M, K, seed=91 + M, outliers=False)
    res = synth.activations(M, K, seed=92 + M, outliers=False)
    y = bl.forward_ex(Wp, gam, rows, x.to(cuda_device), rmsnorm=True, residual=res.to(cuda_device))
    ref = oracle.forward_ex(Wp_ref, g_ref, rows, bits(x), rmsnorm=True, residual=bits(res))
    assert_bf16_exact(bits(y), ref["y"])


@pytest.mark.parametrize("M", [1, 20])
def test_forward_ex_unaligned_segments_take_the_generic_kernel(cuda_device, M):
    K, rows = 256, [40, 24, 8]
    Wp, gam, Wp_ref, g_ref = stacked(rows, K, 95, cuda_device)
    x = synth.activations(M, K, seed=96, outliers=True)
    y, acc = bl.forward_ex(Wp, gam, rows, x.to(cuda_device), rmsnorm=True, want_acc=True)
    ref = oracle.forward_ex(Wp_ref, g_ref, rows, bits(x), rmsnorm=True)
    assert np.array_equal(np_(acc), ref["acc"])
    assert_bf16_exact(bits(y), ref["y"])


@pytest.mark.parametrize("N,K,dtype", [(2560, 2560, "bf16"), (640, 2560, "bf16"), (512, 256, "fp32"),
                                       (3, 12, "bf16"), (136, 196, "fp32")])
def test_pack_rowwise_parity(cuda_device, N, K, dtype):
    W = make_weights(N, K, 0.02, seed=N + K, dtype=dtype)
    Wp, g = bl.pack_weights_rowwise(W.to(cuda_device))
    Wp_ref, g_ref = oracle.pack_weights_rowwise(bits(W) if dtype == "bf16" else np_(W))
    assert np.array_equal(np_(g).view(np.uint32), g_ref.view(np.uint32)), "per-row gamma bits"
    assert np.array_equal(np_(Wp), Wp_ref), "packed bytes"


@pytest.mark.parametrize("M,N,K", [(1, 6912, 2560), (1, 2560, 6912), (4, 640, 2560), (9, 2560, 2560),
                                   (64, 2400, 2560), (300, 640, 4096), (20, 100, 1024), (5, 33, 260)])
def test_forward_rowwise_parity(cuda_device, M, N, K):
    """One gamma per output row: the single-token dp4a GEMV, the fused and unfused
    multi-token GEMV, the tensor-core GEMM (also with split tiles) and the generic kernel."""
    W = make_weights(N, K, 0.02, seed=3 * N + K)
    Wp, g = bl.pack_weights_rowwise(W.to(cuda_device))
    Wp_ref, g_ref = oracle.pack_weights_rowwise(bits(W))
    x = synth.activations(M, K, seed=M + 5, outliers=True)
    res = synth.activations(M, N, seed=M + 6, outliers=False)
    y, acc = bl.forward_rowwise(Wp, g, x.to(cuda_device), residual=res.to(cuda_device), want_acc=True)
    ref = oracle.forward_rowwise(Wp_ref, g_ref, bits(x), residual=bits(res))
    assert np.array_equal(np_(acc), ref["acc"]), "int32 accumulators"
    assert_bf16_exact(bits(y), ref["y"])


def test_forward_largest_k_extreme_codes(cuda_device):
    """K at its documented maximum (262144) with every weight +1 and every code
    127: the field-scaled int32 accumulators of the streamed GEMV reach their
    largest values (128 * 127 * K / 4 < 2^31) and acc = 127 K exactly."""
    K, N, M = 262144, 17, 1
    W = torch.ones((N, K), dtype=torch.bfloat16)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = torch.ones((M, K), dtype=torch.bfloat16)
    y, acc = bl.forward(Wp, gamma, x.to(cuda_device), want_acc=True)
    assert np.all(np_(acc) == 127 * K)
    ref = oracle.forward(Wp_ref, g_ref, bits(x))
    assert np.array_equal(np_(acc), ref["acc"])
    assert_bf16_exact(bits(y), ref["y"])


def test_forward_largest_m(cuda_device):
    """M at its documented maximum (65535 tokens) on the tensor-core path."""
    M, N, K = 65535, 16, 64
    W = make_weights(N, K, 0.02, seed=97)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=98, outliers=True)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device)


def test_forward_misaligned_input_takes_generic_path(cuda_device):
    K, N, M = 256, 64, 20
    W = make_weights(N, K, 0.02, seed=21)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    xb = synth.activations(M, K + 1, seed=22, outliers=True)
    x_dev = xb.to(cuda_device).reshape(-1)[1:1 + M * K].view(M, K)  # 2-byte aligned only
    y, acc = bl.forward(Wp, gamma, x_dev, want_acc=True)
    ref = oracle.forward(Wp_ref, g_ref, bits(x_dev))
    assert np.array_equal(np_(acc), ref["acc"])
    assert_bf16_exact(bits(y), ref["y"])


def test_forward_residual_and_degenerate_tokens(cuda_device):
    K, N, M = 2560, 640, 6
    W = make_weights(N, K, 0.02, seed=5)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=6, outliers=True)
    x[0] = 0                      # all-zero token
    x[1] = x[1] * 1e-8            # below the absmax floor
    x[2, :] = 0
    x[2, 7] = 3.0                 # a single non-zero channel
    res = synth.activations(M, N, seed=8, outliers=False)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device, residual=res)


def test_forward_empty(cuda_device):
    Wp, gamma = bl.pack_weights(make_weights(64, 256, 0.02, seed=1).to(cuda_device))
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=cuda_device)
    y = bl.forward(Wp, gamma, x)
    assert y.shape == (0, 64)


def test_forward_is_deterministic(cuda_device):
    W = make_weights(6912, 2560, 0.02, seed=9).to(cuda_device)
    Wp, gamma = bl.pack_weights(W)
    Wp2, gamma2 = bl.pack_weights(W)
    assert torch.equal(Wp, Wp2) and torch.equal(gamma, gamma2)
    for M in (1, 16, 512):
        x = synth.activations(M, 2560, seed=M).to(cuda_device)
        y1, a1 = bl.forward(Wp, gamma, x, want_acc=True)
        y2, a2 = bl.forward(Wp, gamma, x, want_acc=True)
        assert torch.equal(y1, y2) and torch.equal(a1, a2)


def test_device_error_clean(cuda_device):
    assert bl.get_device_error() == 0


def test_bounded_wait_reports_timeout(cuda_device):
    """A wait that nothing satisfies gives up after its limit, the kernel returns,
    the host sees BL_ERR_TIMEOUT once, and the context keeps working."""
    import ctypes
    BL_ERR_TIMEOUT = 8
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    assert bl.get_device_error() == 0
    assert bl.lib().bitlinear_selftest_timeout(20000, stream) == 0
    assert bl.get_device_error() == BL_ERR_TIMEOUT
    assert bl.get_device_error() == 0
    W = make_weights(64, 256, 0.02, seed=12)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, synth.activations(2, 256, seed=13), cuda_device)


# ----------------------------------------------------------------------------- FFN

def ffn_weights(layer, d, f, dev):
    sg, su, sd = synth.ffn_layer_seeds(layer)
    out = []
    for N, K, seed in ((f, d, sg), (f, d, su), (d, f, sd)):
        W = make_weights(N, K, synth.SIGMA_2B, seed)
        Wp, gamma, Wp_ref, g_ref = pack_both(W, dev)
        out.append((Wp, gamma, Wp_ref, g_ref))
    return out


def test_ffn_chain_decode_teacher_forced(cuda_device):
    """30 layers at d=2560, f=6912, M=1. Each layer's GPU input is fed to the
    oracle, so every layer is compared exactly; the chain is also run end to end."""
    d, f, L = 2560, 6912, 30
    h = synth.activations(1, d, seed=1, outliers=False)
    h_dev = h.to(cuda_device)
    h_ref = bits(h)
    for layer in range(L):
        (Wg, gg, Wgr, ggr), (Wu, gu, Wur, gur), (Wd, gd, Wdr, gdr) = ffn_weights(layer, d, f, cuda_device)
        y_dev = bl.ffn(Wg, gg, Wu, gu, Wd, gd, h_dev, residual=h_dev)
        ref = oracle.ffn_layer(Wgr, ggr, Wur, gur, Wdr, gdr, bits(h_dev), residual=bits(h_dev))
        assert_bf16_close(bits(y_dev), ref["y"], f"layer {layer}")
        assert_bf16_exact(bits(y_dev), ref["y"], f"layer {layer}")
        chain = oracle.ffn_layer(Wgr, ggr, Wur, gur, Wdr, gdr, h_ref, residual=h_ref)
        h_ref = chain["y"]
        h_dev = y_dev
    # end to end: the exact per-layer parity makes the chains identical
    assert_bf16_exact(bits(h_dev), h_ref, "30-layer chain")


def test_ffn_prefill_sampled_tokens(cuda_device):
    """All 30 layers at d=2560, f=6912, M=512, teacher-forced: each layer's GPU
    input rows of the sampled tokens go to the oracle, whose outputs are compared
    bit for bit (tokens are independent, so a sampled row is an exact check)."""
    d, f, M, L = 2560, 6912, 512, 30
    h = synth.activations(M, d, seed=2, outliers=False)
    h_dev = h.to(cuda_device)
    toks = sample_indices(M, 8, seed=4)
    for layer in range(L):
        (Wg, gg, Wgr, ggr), (Wu, gu, Wur, gur), (Wd, gd, Wdr, gdr) = ffn_weights(layer, d, f, cuda_device)
        y_dev = bl.ffn(Wg, gg, Wu, gu, Wd, gd, h_dev, residual=h_dev)
        xin = bits(h_dev)[toks]
        ref = oracle.ffn_layer(Wgr, ggr, Wur, gur, Wdr, gdr, xin, residual=xin)
        got = bits(y_dev)[toks]
        assert_bf16_close(got, ref["y"], f"layer {layer}")
        assert_bf16_exact(got, ref["y"], f"layer {layer}")
        h_dev = y_dev


@pytest.mark.parametrize("M", [2, 4, 8])
def test_ffn_small_batches(cuda_device, M):
    """M <= 4 runs the two-kernel FFN (gate+up with h partials, down with the
    norm and requantisation folded in); M = 8 the unfused decode path."""
    d, f = 2560, 6912
    h = synth.activations(M, d, seed=30 + M, outliers=False)
    h_dev = h.to(cuda_device)
    for layer in range(2):
        (Wg, gg, Wgr, ggr), (Wu, gu, Wur, gur), (Wd, gd, Wdr, gdr) = ffn_weights(layer + 7, d, f, cuda_device)
        y_dev = bl.ffn(Wg, gg, Wu, gu, Wd, gd, h_dev, residual=h_dev)
        ref = oracle.ffn_layer(Wgr, ggr, Wur, gur, Wdr, gdr, bits(h_dev), residual=bits(h_dev))
        assert_bf16_close(bits(y_dev), ref["y"], f"M={M} layer {layer}")
        assert_bf16_exact(bits(y_dev), ref["y"], f"M={M} layer {layer}")
        h_dev = y_dev


def test_ffn_stream_k_fp32_projections(cuda_device):
    """M = 40 at d = 4096, f = 1024: gate and up run on the tensor cores with
    split tiles and fp32 outputs (the fix-up's fp32 store), down unsplit."""
    d, f, M = 4096, 1024, 40
    Wg, Wu, Wd = (make_weights(f, d, 0.02, 41), make_weights(f, d, 0.02, 42), make_weights(d, f, 0.02, 43))
    P = [pack_both(W, cuda_device) for W in (Wg, Wu, Wd)]
    x = synth.activations(M, d, seed=44, outliers=True)
    y = bl.ffn(P[0][0], P[0][1], P[1][0], P[1][1], P[2][0], P[2][1], x.to(cuda_device), residual=x.to(cuda_device))
    ref = oracle.ffn_layer(P[0][2], P[0][3], P[1][2], P[1][3], P[2][2], P[2][3], bits(x), residual=bits(x))
    assert_bf16_close(bits(y), ref["y"])
    assert_bf16_exact(bits(y), ref["y"])


def test_ffn_small_ragged(cuda_device):
    d, f, M = 64, 200, 3
    Wg, Wu, Wd = (make_weights(f, d, 0.02, 1), make_weights(f, d, 0.02, 2), make_weights(d, f, 0.02, 3))
    P = [pack_both(W, cuda_device) for W in (Wg, Wu, Wd)]
    x = synth.activations(M, d, seed=3, outliers=True)
    y = bl.ffn(P[0][0], P[0][1], P[1][0], P[1][1], P[2][0], P[2][1], x.to(cuda_device))
    ref = oracle.ffn_layer(P[0][2], P[0][3], P[1][2], P[1][3], P[2][2], P[2][3], bits(x))
    assert_bf16_exact(bits(y), ref["y"])


@pytest.mark.parametrize("M,d,f", [(1, 6912, 2560), (1, 12288, 1024), (1, 2560, 12288), (2, 6912, 2560),
                                   (3, 6912, 2560), (4, 8192, 1024)])
def test_ffn_fused_prologue_routes(cuda_device, M, d, f):
    """The two-kernel FFN (up to 4 tokens) with each of its quantiser forms:
    gate+up with 2 and 8 register groups for one token (d = 6912, 12288), with two
    groups for two tokens (d = 6912), and the two-pass loop for three and four
    tokens with d > 4096; the down projection's one-token form for f <= 8192 and
    its two-pass loop beyond (f = 12288)."""
    Wg, Wu, Wd = (make_weights(f, d, 0.02, 7100 + d), make_weights(f, d, 0.02, 7200 + d),
                  make_weights(d, f, 0.02, 7300 + f))
    P = [pack_both(W, cuda_device) for W in (Wg, Wu, Wd)]
    x = synth.activations(M, d, seed=7400 + M, outliers=True)
    res = synth.activations(M, d, seed=7500 + M, outliers=False)
    y = bl.ffn(P[0][0], P[0][1], P[1][0], P[1][1], P[2][0], P[2][1], x.to(cuda_device),
               residual=res.to(cuda_device))
    ref = oracle.ffn_layer(P[0][2], P[0][3], P[1][2], P[1][3], P[2][2], P[2][3], bits(x), residual=bits(res))
    assert_bf16_close(bits(y), ref["y"])
    assert_bf16_exact(bits(y), ref["y"])
    assert bl.get_device_error() == 0


# ----------------------------------------------------------------------------- tensor-core GEMV (M <= 16)

@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560), (2560, 640), (256, 136), (768, 17), (8192, 1000)])
def test_forward_gemv_tensor_core(cuda_device, K, N, M):
    """The tcgen05 GEMV (weights unpacked into tensor memory, tokens as the MMA's
    N = 8 / 16), forced on: ragged N, K with a half last stage (6912 = 13.5 x 512),
    K split over clusters of 1 to 8 CTAs, residual and the int32 dump."""
    W = make_weights(N, K, 0.02, seed=4000 + K + N)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=4100 + M, outliers=True)
    res = synth.activations(M, N, seed=4200 + M, outliers=False)
    with bl.gemv_kernel(bl.BL_GEMV_TENSOR):
        check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device, residual=res)
    assert bl.get_device_error() == 0


@pytest.mark.parametrize("M", [1, 16])
@pytest.mark.parametrize("K,N", [(8192, 28672), (28672, 8192)])
def test_forward_gemv_tensor_core_100b_sampled(cuda_device, K, N, M):
    W = make_weights(N, K, synth.SIGMA_100B, seed=4300 + K)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=4400 + M, outliers=True)
    rows = sample_indices(N, 256, seed=M + 11)
    with bl.gemv_kernel(bl.BL_GEMV_TENSOR):
        check_forward_sampled(Wp, gamma, Wp_ref, g_ref, x, cuda_device, rows, np.arange(M))


@pytest.mark.parametrize("M", [2, 12])
def test_forward_gemv_tensor_core_rowwise_and_segments(cuda_device, M):
    K, N = 2560, 1024
    W = make_weights(N, K, 0.02, seed=4500)
    Wp, g = bl.pack_weights_rowwise(W.to(cuda_device))
    Wp_ref, g_ref = oracle.pack_weights_rowwise(bits(W))
    x = synth.activations(M, K, seed=4501 + M, outliers=True)
    with bl.gemv_kernel(bl.BL_GEMV_TENSOR):
        y, acc = bl.forward_rowwise(Wp, g, x.to(cuda_device), want_acc=True)
    ref = oracle.forward_rowwise(Wp_ref, g_ref, bits(x))
    assert np.array_equal(np_(acc), ref["acc"])
    assert_bf16_exact(bits(y), ref["y"])
    rows = [512, 256, 256]
    parts = [make_weights(n, K, 0.02, seed=4510 + i) for i, n in enumerate(rows)]
    dev_parts = [bl.pack_weights(p.to(cuda_device)) for p in parts]
    ref_parts = [oracle.pack_weights(bits(p)) for p in parts]
    with bl.gemv_kernel(bl.BL_GEMV_TENSOR):
        yq = bl.forward_ex(torch.cat([p[0] for p in dev_parts]), torch.cat([p[1].reshape(1) for p in dev_parts]),
                           rows, x.to(cuda_device), rmsnorm=True)
    rq = oracle.forward_ex(np.concatenate([p[0] for p in ref_parts]), [p[1] for p in ref_parts], rows, bits(x),
                           rmsnorm=True)
    assert_bf16_exact(bits(yq), rq["y"])


@pytest.mark.parametrize("M", [4, 16])
def test_ffn_gemv_tensor_core(cuda_device, M):
    """FFN projections on the tensor-core GEMV (fp32 gate/up outputs, then the
    requantised down projection with the residual)."""
    d, f = 2560, 6912
    h = synth.activations(M, d, seed=4600 + M, outliers=False)
    (Wg, gg, Wgr, ggr), (Wu, gu, Wur, gur), (Wd, gd, Wdr, gdr) = ffn_weights(11, d, f, cuda_device)
    with bl.gemv_kernel(bl.BL_GEMV_TENSOR):
        y = bl.ffn(Wg, gg, Wu, gu, Wd, gd, h.to(cuda_device), residual=h.to(cuda_device))
    ref = oracle.ffn_layer(Wgr, ggr, Wur, gur, Wdr, gdr, bits(h), residual=bits(h))
    assert_bf16_exact(bits(y), ref["y"])


def test_gemv_kernel_choice_gives_the_same_bits(cuda_device):
    """Every M <= 16 kernel computes the same integers and bf16 bits."""
    K, N, M = 6912, 2560, 6
    W = make_weights(N, K, 0.02, seed=4700)
    Wp, gamma = bl.pack_weights(W.to(cuda_device))
    x = synth.activations(M, K, seed=4701, outliers=True).to(cuda_device)
    outs = []
    for kind in (bl.BL_GEMV_STREAM, bl.BL_GEMV_TENSOR, bl.BL_GEMV_LUT, bl.BL_GEMV_AUTO):
        with bl.gemv_kernel(kind):
            y, acc = bl.forward(Wp, gamma, x, want_acc=True)
        outs.append((bits(y), np_(acc)))
    for y, acc in outs[1:]:
        assert np.array_equal(acc, outs[0][1]) and np.array_equal(y, outs[0][0])


# ----------------------------------------------------------------------------- lookup-table GEMV (M <= 16)

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 16])
@pytest.mark.parametrize("K,N", [(2560, 6912), (6912, 2560), (2560, 640), (256, 136), (13056, 33)])
def test_forward_gemv_lookup_table(cuda_device, K, N, M):
    """The T-MAC-style lookup-table GEMV, forced on: table segments of 128-768
    words with a partial last chunk (K = 2560: 160 words; 6912: 432), several
    segments (K = 13056 at one token: 816 words), one to four launches of up to
    four tokens, residual and the int32 dump."""
    W = make_weights(N, K, 0.02, seed=5000 + K + N)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=5100 + M, outliers=True)
    res = synth.activations(M, N, seed=5200 + M, outliers=False)
    with bl.gemv_kernel(bl.BL_GEMV_LUT):
        check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device, residual=res)
    assert bl.get_device_error() == 0


@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("K,N", [(8192, 28672), (28672, 8192)])
def test_forward_gemv_lookup_table_100b_sampled(cuda_device, K, N, M):
    W = make_weights(N, K, synth.SIGMA_100B, seed=5300 + K)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(M, K, seed=5400 + M, outliers=True)
    rows = sample_indices(N, 256, seed=M + 13)
    with bl.gemv_kernel(bl.BL_GEMV_LUT):
        check_forward_sampled(Wp, gamma, Wp_ref, g_ref, x, cuda_device, rows, np.arange(M))


def test_forward_gemv_lookup_table_rowwise(cuda_device):
    K, N, M = 2560, 1000, 3
    W = make_weights(N, K, 0.02, seed=5500)
    Wp, g = bl.pack_weights_rowwise(W.to(cuda_device))
    Wp_ref, g_ref = oracle.pack_weights_rowwise(bits(W))
    x = synth.activations(M, K, seed=5501, outliers=True)
    with bl.gemv_kernel(bl.BL_GEMV_LUT):
        y, acc = bl.forward_rowwise(Wp, g, x.to(cuda_device), want_acc=True)
    ref = oracle.forward_rowwise(Wp_ref, g_ref, bits(x))
    assert np.array_equal(np_(acc), ref["acc"])
    assert_bf16_exact(bits(y), ref["y"])


# ----------------------------------------------------------------------------- one token, long rows

@pytest.mark.parametrize("K", [4608, 8192, 12288, 20480, 32768, 36864])
@pytest.mark.parametrize("N", [1001, 300])
def test_forward_single_token_long_rows(cuda_device, K, N):
    """M = 1 on the streamed dp4a GEMV with units of whole rows (16 rows up to
    2 KiB per row, 8 up to 4 KiB, 4 beyond; two K segments past 8 KiB) and the
    register-resident quantiser for 8192 <= K <= 32768; N ragged for every unit
    height."""
    W = make_weights(N, K, 0.01, seed=6000 + K + N)
    Wp, gamma, Wp_ref, g_ref = pack_both(W, cuda_device)
    x = synth.activations(1, K, seed=6100 + K, outliers=True)
    res = synth.activations(1, N, seed=6200 + N, outliers=False)
    check_forward_full(Wp, gamma, Wp_ref, g_ref, x, cuda_device, residual=res)


@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("norm", [False, True])
def test_forward_ex_two_tokens_register_quantiser(cuda_device, M, norm):
    """One or two tokens with 4096 < K <= 8192 on the extended calls: the
    in-kernel quantiser that keeps both tokens' x in registers (two groups of 16
    per thread), with and without the RMSNorm, for stacked segments with their own
    gammas and for one gamma per row."""
    K, rows = 6912, [1024, 256, 256]
    Wp, gam, Wp_ref, g_ref = stacked(rows, K, 97, cuda_device)
    x = synth.activations(M, K, seed=98 + M, outliers=True)
    y, acc = bl.forward_ex(Wp, gam, rows, x.to(cuda_device), rmsnorm=norm, want_acc=True)
    ref = oracle.forward_ex(Wp_ref, g_ref, rows, bits(x), rmsnorm=norm)
    assert np.array_equal(np_(acc), ref["acc"]), "int32 accumulators"
    assert_bf16_exact(bits(y), ref["y"])
    if not norm:
        W = make_weights(1000, K, 0.02, seed=99)
        Wr, gr = bl.pack_weights_rowwise(W.to(cuda_device))
        Wr_ref, gr_ref = oracle.pack_weights_rowwise(bits(W))
        res = synth.activations(M, 1000, seed=100 + M, outliers=False)
        y, acc = bl.forward_rowwise(Wr, gr, x.to(cuda_device), residual=res.to(cuda_device), want_acc=True)
        ref = oracle.forward_rowwise(Wr_ref, gr_ref, bits(x), residual=bits(res))
        assert np.array_equal(np_(acc), ref["acc"])
        assert_bf16_exact(bits(y), ref["y"])
    assert bl.get_device_error() == 0


@pytest.mark.parametrize("K", [12288, 28672])
def test_forward_ex_single_token_long_rows_rmsnorm(cuda_device, K):
    rows = [256, 64, 64]
    parts = [make_weights(n, K, 0.01, seed=6300 + i) for i, n in enumerate(rows)]
    dev_parts = [bl.pack_weights(p.to(cuda_device)) for p in parts]
    ref_parts = [oracle.pack_weights(bits(p)) for p in parts]
    x = synth.activations(1, K, seed=6310, outliers=True)
    yq = bl.forward_ex(torch.cat([p[0] for p in dev_parts]), torch.cat([p[1].reshape(1) for p in dev_parts]),
                       rows, x.to(cuda_device), rmsnorm=True)
    rq = oracle.forward_ex(np.concatenate([p[0] for p in ref_parts]), [p[1] for p in ref_parts], rows, bits(x),
                           rmsnorm=True)
    assert_bf16_exact(bits(yq), rq["y"])


# ----------------------------------------------------------------------------- FFN, gate+up in one tensor-core launch

@pytest.mark.parametrize("M,d,f", [(17, 256, 200), (40, 512, 1000), (300, 2560, 6912), (129, 4096, 1024)])
def test_ffn_dual_gemm(cuda_device, M, d, f):
    """M > 16: gate and up in one launch (128 + 128 weight rows per tile) whose
    epilogue forms h and the per-tile sum h^2 / max |h|; then the requantisation
    from those partials and the down projection (generic kernel for f = 200 and
    1000, tensor cores otherwise). f = 200 and 1000 leave a partial last tile."""
    Wg, Wu, Wd = (make_weights(f, d, 0.02, 7000 + d), make_weights(f, d, 0.02, 7001 + d),
                  make_weights(d, f, 0.02, 7002 + d))
    P = [pack_both(W, cuda_device) for W in (Wg, Wu, Wd)]
    x = synth.activations(M, d, seed=7003 + M, outliers=False)
    y = bl.ffn(P[0][0], P[0][1], P[1][0], P[1][1], P[2][0], P[2][1], x.to(cuda_device), residual=x.to(cuda_device))
    ref = oracle.ffn_layer(P[0][2], P[0][3], P[1][2], P[1][3], P[2][2], P[2][3], bits(x), residual=bits(x))
    assert_bf16_exact(bits(y), ref["y"])
    assert bl.get_device_error() == 0

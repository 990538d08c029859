"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against a hand-worked example, a closed form, an
invariant, a brute force over every case, or a library routine, chosen so that a
plausible slip (a dropped eps, a wrong bit order, a transposed operand, a wrong
rounding mode, a dropped ReLU or square) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from bitlinear_w1_a8_02_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------- bf16

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        rng.standard_normal(2000).astype(np.float32) * np.float32(1e-30),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38, 1e-45], np.float32),
    ])
    # exact ties: low 16 bits == 0x8000, both parities of the kept part
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    vals = np.concatenate([vals, ties, -ties]).astype(np.float32)
    ours = oracle.f32_to_bf16(vals)
    ref = bf16_bits(torch.from_numpy(vals).to(torch.bfloat16))
    assert np.array_equal(ours, ref)
    # NaNs whose payload sits only in the low half, or that rounding up would carry
    # into the sign, stay NaNs of the same sign (exponent all ones, mantissa not 0)
    nans = np.array([0x7F800001, 0xFF800001, 0x7FFFFFFF, 0xFFFFFFFF, 0x7FC00000], np.uint32).view(np.float32)
    out = oracle.f32_to_bf16(nans).astype(np.uint32)
    assert np.all((out & 0x7F80) == 0x7F80) and np.all((out & 0x007F) != 0)
    assert (out >> 15).tolist() == [0, 1, 0, 1, 0]
    assert np.all(np.isnan(torch.from_numpy(nans).to(torch.bfloat16).float().numpy()))
    back = oracle.bf16_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float().numpy())


# ----------------------------------------------------------------------------- packing

def test_pack_unpack_all_ternary_quads():
    quads = np.array(np.meshgrid(*([[-1, 0, 1]] * 4), indexing="ij")).reshape(4, -1).T.astype(np.int8)
    assert quads.shape == (81, 4)
    Wp = oracle.pack(quads)
    q, bad = oracle.unpack(Wp, 4)
    assert bad == 0
    assert np.array_equal(q, quads)
    assert len(set(Wp[:, 0].tolist())) == 81


def test_pack_bit_order_and_code_offset():
    # weight i of a byte sits in bits 2i..2i+1 as code q+1
    cases = {
        (0, 0, 0, 0): 0x55, (-1, -1, -1, -1): 0x00, (1, 1, 1, 1): 0xAA,
        (1, 0, 0, 0): 0x56, (0, 0, 0, 1): 0x95, (-1, 0, 0, 0): 0x54, (0, -1, 0, 0): 0x51,
    }
    for quad, byte in cases.items():
        assert oracle.pack(np.array([quad], np.int8))[0, 0] == byte, quad
    # second byte of a row holds weights 4..7
    q = np.zeros((1, 8), np.int8)
    q[0, 5] = 1
    assert oracle.pack(q).tolist() == [[0x55, 0x59]]


def test_unpack_all_bytes():
    Wp = np.arange(256, dtype=np.uint8).reshape(256, 1)
    q, bad = oracle.unpack(Wp, 4)
    fields = [(b >> (2 * i)) & 3 for b in range(256) for i in range(4)]
    assert bad == sum(f == 3 for f in fields)
    valid = [b for b in range(256) if all(((b >> (2 * i)) & 3) != 3 for i in range(4))]
    assert len(valid) == 81
    assert set(np.unique(q[valid]).tolist()) == {-1, 0, 1}


# ----------------------------------------------------------------------------- worked example

def test_worked_4x4_example():
    g = json.load(open(os.path.join(GOLDEN, "worked_4x4.json")))
    W = np.array(g["W"], np.float32)
    gamma = oracle.absmean(W)
    assert gamma == np.float32(g["gamma"])
    q = oracle.ternarize(W, gamma)
    assert q.tolist() == g["q"]
    Wp, gamma2 = oracle.pack_weights(W)
    assert gamma2 == gamma
    assert Wp[:, 0].tolist() == g["packed"]
    x = np.array(g["x"], np.float32)
    xq, s, xs = oracle.quant_act(x)
    assert xq.tolist() == g["xq"]
    assert s.tolist() == np.array(g["s"], np.float32).tolist()
    assert xs.tolist() == g["xsum"]
    acc = oracle.int_gemm_packed(Wp, xq)
    assert acc.tolist() == g["acc"]
    y, y32 = oracle.dequant(acc, gamma, s, want_f32=True)
    assert y32.tolist() == np.array(g["y32"], np.float32).tolist()
    assert np.array_equal(y, bf16_bits(torch.tensor(g["y32"], dtype=torch.float32).to(torch.bfloat16)))
    # the whole forward reaches the same values from bf16 inputs
    out = oracle.forward(Wp, gamma, bf16_bits(torch.tensor(g["x"]).to(torch.bfloat16)))
    assert out["acc"].tolist() == g["acc"]
    assert np.array_equal(out["y"], y)
    assert out["xq"].tolist() == g["xq"] and out["xsum"].tolist() == g["xsum"]
    assert out["s"].tolist() == np.array(g["s"], np.float32).tolist()


# ----------------------------------------------------------------------------- weights

def test_ternarize_eps_and_half_even():
    # mean |W| = 1/4 exactly; w0 / gamma = 0.5 + 2^-18 would round to 1 without
    # the eps, but w0 / (gamma + 1e-5) < 0.5 rounds to 0.
    W = np.array([[0.125 + 2.0 ** -20, 0.375 - 2.0 ** -20, 0.25, 0.25]], np.float32)
    gamma = oracle.absmean(W)
    assert gamma == np.float32(0.25)
    assert oracle.ternarize(W, gamma).tolist() == [[0, 1, 1, 1]]
    # exact halves of d round to even: 0.5 d -> 0, -0.5 d -> 0, 1.5 d -> 2 -> clip 1
    d = np.float32(np.float32(0.25) + np.float32(1e-5))
    W2 = np.array([0.5 * d, -0.5 * d, 1.5 * d, -1.5 * d, 2.5 * d, 0.0], np.float32)
    assert np.array_equal(W2 / d, np.array([0.5, -0.5, 1.5, -1.5, 2.5, 0.0], np.float32))
    assert oracle.ternarize(W2, np.float32(0.25)).tolist() == [0, 0, 1, -1, 1, 0]


def test_absmean_closed_forms():
    assert oracle.absmean(np.full(1000, -0.375, np.float32)) == np.float32(0.375)
    W = (np.arange(1, 4097, dtype=np.float32) * np.float32(2.0 ** -12)) * np.where(np.arange(4096) % 2, 1, -1)
    exact = math.fsum(abs(float(v)) for v in W) / W.size
    assert oracle.absmean(W.astype(np.float32)) == np.float32(exact)
    # one rounding, of the fp64 quotient: sum = 3 + 5 * 2^-23 (exact in fp64), and
    # sum / 3 = 1 + (5/3) 2^-23 rounds to 1 + 2 * 2^-23. Rounding the sum to fp32
    # first would give 3 + 4 * 2^-23 (a tie, to even), then 1 + 2^-23.
    W3 = np.array([1.0, 1.0, 1.0 + 5 * 2.0 ** -23], np.float32)
    assert oracle.absmean(W3) == np.float32(1.0 + 2.0 ** -22)
    # all-zero W: gamma = 0, every code 0
    Z = np.zeros((3, 8), np.float32)
    Wp, g = oracle.pack_weights(Z)
    assert g == 0.0 and np.all(Wp == 0x55)


def test_gaussian_ternary_statistics():
    # For W ~ N(0, sigma^2): gamma -> sigma*sqrt(2/pi), P(q = 0) = P(|Z| < sqrt(2/pi)/2)
    sigma = synth.SIGMA_2B
    W = synth.weights(1024, 4096, sigma, seed=7, dtype="fp32").numpy()
    n = W.size
    gamma = oracle.absmean(W)
    g_exp = sigma * math.sqrt(2 / math.pi)
    assert abs(gamma / g_exp - 1) < 5 * 0.756 / math.sqrt(n)
    q = oracle.ternarize(W, gamma)
    p0 = math.erf(math.sqrt(2 / math.pi) / 2 / math.sqrt(2))
    assert abs(p0 - 0.31006) < 1e-4
    frac0 = float(np.mean(q == 0))
    assert abs(frac0 - p0) < 5 * math.sqrt(p0 * (1 - p0) / n) + 1e-4
    pp = (1 - p0) / 2
    assert abs(float(np.mean(q == 1)) - pp) < 5 * math.sqrt(pp * (1 - pp) / n) + 1e-4


# ----------------------------------------------------------------------------- activations

def test_quant_act_half_even_and_range():
    # amax = 127 -> s = 1 exactly, so xq = rint(x) with ties to even
    x = np.array([[127.0, 62.5, 63.5, 2.5, -0.5, 1.5, -2.5, -127.0]], np.float32)
    xq, s, xs = oracle.quant_act(x)
    assert s[0] == 1.0
    assert xq.tolist() == [[127, 62, 64, 2, 0, 2, -2, -127]]
    assert xs[0] == sum(xq[0].tolist())


def test_quant_act_invariants():
    x = synth.activations(64, 2560, seed=1, outliers=True).float().numpy()
    x[5] = 0.0
    xq, s, xs = oracle.quant_act(x)
    nz = np.abs(x).max(axis=1) > 0
    assert np.all(np.abs(xq[nz]).max(axis=1) == 127)
    assert xq.min() >= -127 and xq.max() <= 127
    assert np.all(xq[5] == 0) and s[5] == np.float32(127.0) / np.float32(1e-5)
    assert np.array_equal(xs, xq.astype(np.int64).sum(axis=1))
    # scaling a token by a power of two leaves the codes unchanged
    for p in (-3, 4):
        xq2, s2, _ = oracle.quant_act(x * np.float32(2.0 ** p))
        assert np.array_equal(xq2, xq)
        assert np.array_equal(s2[nz], s[nz] * np.float32(2.0 ** -p))


def test_quant_act_tiny_token_uses_floor():
    # amax = 1e-6 < 1e-5: s = 127 / 1e-5, so the largest code is 13, not 127
    x = np.array([[1e-6, -5e-7, 0.0, 2.5e-7]], np.float32)
    xq, s, _ = oracle.quant_act(x)
    assert s[0] == np.float32(127.0) / np.float32(1e-5)
    assert xq.tolist() == [[13, -6, 0, 3]]


# ----------------------------------------------------------------------------- contraction

@pytest.mark.parametrize("M,N,K", [(1, 1, 4), (3, 5, 8), (7, 3, 32), (8, 8, 12), (2, 17, 64)])
def test_int_gemm_matches_numpy(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    q = rng.integers(-1, 2, (N, K)).astype(np.int8)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    ref = xq.astype(np.int64) @ q.astype(np.int64).T
    acc = oracle.int_gemm(q, xq)
    assert acc.shape == (M, N)
    assert np.array_equal(acc, ref)
    assert np.array_equal(oracle.int_gemm_packed(oracle.pack(q), xq), ref)


def test_int_gemm_special_cases():
    rng = np.random.default_rng(3)
    xq = rng.integers(-127, 128, (4, 40)).astype(np.int8)
    rows = xq.astype(np.int64).sum(axis=1)
    for c, expect in ((1, rows), (-1, -rows), (0, 0 * rows)):
        q = np.full((6, 40), c, np.int8)
        acc = oracle.int_gemm_packed(oracle.pack(q), xq)
        assert np.array_equal(acc, np.repeat(expect[:, None], 6, axis=1))
    # extreme magnitude: K = 28672 with every code and activation at its limit
    K = 28672
    q = np.ones((1, K), np.int8)
    xq = np.full((1, K), -127, np.int8)
    assert oracle.int_gemm_packed(oracle.pack(q), xq)[0, 0] == -127 * K


# ----------------------------------------------------------------------------- dequant

def test_dequant_exact_and_residual():
    acc = np.array([[4, -8, 0, 3]], np.int32)
    s = np.array([2.0], np.float32)
    y, y32 = oracle.dequant(acc, np.float32(0.5), s, want_f32=True)
    assert y32.tolist() == [[1.0, -2.0, 0.0, 0.75]]
    res = bf16_bits(torch.tensor([[1.0, 1.0, -3.0, 256.0]]).to(torch.bfloat16))
    y, y32 = oracle.dequant(acc, np.float32(0.5), s, residual=res, want_f32=True)
    assert y32.tolist() == [[2.0, -1.0, -3.0, 256.75]]
    # bf16 keeps 8 significant bits: 256.75 rounds to 256 (tie-free, nearest)
    assert oracle.bf16_to_f32(y).tolist() == [[2.0, -1.0, -3.0, 256.0]]


# ----------------------------------------------------------------------------- FFN

def test_relu2_gate_values():
    assert oracle.relu2_gate(2.0, 3.0) == 12.0
    assert oracle.relu2_gate(-2.0, 3.0) == 0.0
    assert oracle.relu2_gate(0.5, -4.0) == -1.0
    # The square is rounded to fp32 before u multiplies it. With t = 1 + 2^-12 the
    # exact square 1 + 2^-11 + 2^-24 lies halfway between two fp32 values and rounds
    # to the even one, 1 + 2^-11; times u = 1 + 2^-11 that is 1 + 2^-10 + 2^-22,
    # exact. Multiplying t * (t * u), or rounding the exact triple product once,
    # gives 1 + 2^-10 + 2^-22 + 2^-23 instead.
    assert oracle.relu2_gate(1 + 2.0 ** -12, 1 + 2.0 ** -11) == 1 + 2.0 ** -10 + 2.0 ** -22


def test_subln_rms_closed_form():
    h = np.array([3.0, -4.0, 0.0, 0.0], np.float32)  # mean h^2 = 6.25
    r, hn = oracle.subln_rms(h)
    assert abs(float(r) - 1 / math.sqrt(6.25 + 1e-5)) < 1e-7
    hb = synth.activations(1, 6912, seed=4, outliers=False).float().numpy()[0] * np.float32(1e-3)
    r, hn = oracle.subln_rms(hb)
    ms = float(np.mean(hb.astype(np.float64) ** 2))
    assert abs(float(r) / (1 / math.sqrt(ms + 1e-5)) - 1) < 1e-6
    assert abs(float(np.mean(hn.astype(np.float64) ** 2)) - ms / (ms + 1e-5)) < 1e-5


def _packed_rows(codes):
    return oracle.pack(np.array(codes, np.int8))


def test_ffn_structured_closed_form():
    """Gate rows with j+1 leading +1 codes, up and down all +1, constant x.

    g_j = (j+1) * gg * c, u_j = d * gu * c, h_j = ((j+1) gg c)^2 d gu c.
    hn_j = h_j / sqrt(mean h^2 + eps); q2_j = rint(127 h_j / h_max);
    y_n = res + gd * sum_j q2_j * hn_max / 127 for every output n.
    A dropped ReLU, square, mean or eps moves y far outside bf16 rounding.
    """
    d, f = 16, 8
    gg, gu, gd = np.float32(0.5), np.float32(0.25), np.float32(0.125)
    Wg = _packed_rows([[1] * (j + 1) + [0] * (d - j - 1) for j in range(f)])
    Wu = _packed_rows([[1] * d for _ in range(f)])
    Wd = _packed_rows([[1] * f for _ in range(d)])
    for c, res_val in ((0.0625, 1.0), (0.001, 0.0)):
        x = bf16_bits(torch.full((1, d), c).to(torch.bfloat16))
        res = bf16_bits(torch.full((1, d), res_val).to(torch.bfloat16))
        out = oracle.ffn_layer(Wg, gg, Wu, gu, Wd, gd, x, residual=res)
        cb = float(torch.tensor(c).to(torch.bfloat16))
        g = np.array([(j + 1) * gg * cb for j in range(f)], np.float64)
        u = d * gu * cb
        h = g ** 2 * u
        hn = h / math.sqrt(np.mean(h ** 2) + 1e-5)
        q2 = np.rint(127 * h / h.max())
        y = res_val + gd * q2.sum() * hn.max() / 127
        assert np.array_equal(out["q2"][0], q2.astype(np.int8))
        got = oracle.bf16_to_f32(out["y"])[0]
        assert np.all(np.abs(got - y) <= 2.0 ** -8 * abs(y) + 1e-30), (got, y)


def test_ffn_negative_gate_is_cut():
    d, f = 8, 8
    Wg = _packed_rows([[1] * d] * f)
    Wd = _packed_rows([[1] * f] * d)
    x = bf16_bits(torch.full((1, d), -0.5).to(torch.bfloat16))
    res = bf16_bits(torch.full((1, d), 0.75).to(torch.bfloat16))
    out = oracle.ffn_layer(Wg, 1.0, Wg, 1.0, Wd, 1.0, x, residual=res)
    assert np.all(out["h"] == 0) and np.all(out["q2"] == 0)
    assert np.all(oracle.bf16_to_f32(out["y"]) == 0.75)


def test_ffn_requant_tracks_unnormalised_codes():
    # RMSNorm is a positive per-token rescale, so requantising hn gives the codes
    # of h itself except at rare rounding ties.
    rng_seed = 11
    d, f, M = 256, 512, 8
    W = [synth.weights(f, d, 0.02, rng_seed + i) for i in range(2)] + [synth.weights(d, f, 0.02, rng_seed + 2)]
    packed = [oracle.pack_weights(bf16_bits(w)) for w in W]
    x = bf16_bits(synth.activations(M, d, seed=rng_seed, outliers=True))
    out = oracle.ffn_layer(packed[0][0], packed[0][1], packed[1][0], packed[1][1],
                           packed[2][0], packed[2][1], x, residual=x)
    q_direct, _, _ = oracle.quant_act(out["h"])
    mismatch = np.mean(q_direct != out["q2"])
    assert mismatch < 1e-3
    assert np.all(np.abs(q_direct.astype(int) - out["q2"].astype(int)) <= 1)


# ----------------------------------------------------------------------------- stacked projections

def test_forward_ex_structured_closed_form():
    """Two stacked matrices with their own gamma, constant input.

    Segment 0 row j has j+1 leading +1 codes, segment 1 rows are all -1; a constant
    token c quantises to 127 everywhere, so acc = 127 (j+1) and -127 K, and
    y = acc * gamma_i * a / 127 with a = c, or a = c r after the unit-weight
    RMSNorm (r = 1 / sqrt(c^2 + eps)). A swapped gamma, a missing norm or a sum in
    place of the mean moves y far outside bf16 rounding.
    """
    K, n0, n1 = 16, 6, 3
    g = np.array([0.5, 0.25], np.float32)
    W0 = _packed_rows([[1] * (j + 1) + [0] * (K - j - 1) for j in range(n0)])
    W1 = _packed_rows([[-1] * K for _ in range(n1)])
    Wp = np.concatenate([W0, W1])
    for c, res_val, norm in ((0.0625, 0.0, False), (0.0625, 1.5, True), (3.0, -2.0, True)):
        x = bf16_bits(torch.full((1, K), c).to(torch.bfloat16))
        res = bf16_bits(torch.full((1, n0 + n1), res_val).to(torch.bfloat16))
        out = oracle.forward_ex(Wp, g, [n0, n1], x, rmsnorm=norm, residual=res)
        cb = float(torch.tensor(c).to(torch.bfloat16))
        a = cb / math.sqrt(cb * cb + 1e-5) if norm else cb
        acc = [127 * (j + 1) for j in range(n0)] + [-127 * K] * n1
        gam = [float(g[0])] * n0 + [float(g[1])] * n1
        assert out["acc"][0].tolist() == acc
        term = np.array([acc[n] * gam[n] * a / 127 for n in range(n0 + n1)])
        y = res_val + term
        got = oracle.bf16_to_f32(out["y"])[0].astype(np.float64)
        # one bf16 rounding of the sum, plus fp32 roundings far below it
        assert np.all(np.abs(got - y) <= 2.0 ** -8 * (np.abs(res_val) + np.abs(term))), (norm, got, y)


def test_forward_ex_segments_are_the_separate_projections():
    K, M = 256, 5
    Ws = [synth.weights(n, K, 0.02, 70 + i) for i, n in enumerate((48, 16, 32))]
    packed = [oracle.pack_weights(bf16_bits(w)) for w in Ws]
    x = bf16_bits(synth.activations(M, K, seed=71, outliers=True))
    res = bf16_bits(synth.activations(M, 96, seed=72, outliers=False))
    out = oracle.forward_ex(np.concatenate([p[0] for p in packed]), [p[1] for p in packed], [48, 16, 32], x,
                            residual=res)
    col = 0
    for (Wp, gamma), n in zip(packed, (48, 16, 32)):
        ref = oracle.forward(Wp, gamma, x, residual=np.ascontiguousarray(res[:, col:col + n]))
        assert np.array_equal(out["acc"][:, col:col + n], ref["acc"])
        assert np.array_equal(out["y"][:, col:col + n], ref["y"])
        col += n


def test_forward_ex_rmsnorm_only_rescales_the_codes():
    # The RMSNorm is a positive per-token rescale: the codes (so acc) are those of
    # x itself except at rare rounding ties.
    K, N, M = 512, 64, 16
    Wp, gamma = oracle.pack_weights(bf16_bits(synth.weights(N, K, 0.02, 73)))
    x = bf16_bits(synth.activations(M, K, seed=74, outliers=True))
    plain = oracle.forward_ex(Wp, [gamma], [N], x, rmsnorm=False)
    normed = oracle.forward_ex(Wp, [gamma], [N], x, rmsnorm=True)
    diff = np.abs(plain["acc"].astype(np.int64) - normed["acc"].astype(np.int64))
    assert np.mean(diff != 0) < 0.05 and np.all(diff <= 3 * 2)


# ----------------------------------------------------------------------------- per-row gamma variant

def test_rowwise_worked_2x4():
    g = json.load(open(os.path.join(GOLDEN, "rowwise_2x4.json")))
    W = np.array(g["W"], np.float32)
    Wp, gam = oracle.pack_weights_rowwise(W)
    assert gam.tolist() == g["gammas"]
    q, bad = oracle.unpack(Wp, 4)
    assert bad == 0 and q.tolist() == g["q"]
    assert Wp.tolist() == g["packed"]
    Wp_t, gam_t = oracle.pack_weights(W)
    assert float(gam_t) == g["per_tensor_gamma"]
    assert oracle.unpack(Wp_t, 4)[0][1].tolist() == g["per_tensor_q_row1"]


def test_rowwise_single_row_is_per_tensor():
    W = bf16_bits(synth.weights(1, 2560, 0.02, 61))
    Wp_r, g_r = oracle.pack_weights_rowwise(W)
    Wp_t, g_t = oracle.pack_weights(W)
    assert np.array_equal(Wp_r, Wp_t) and g_r[0] == g_t


def test_rowwise_power_of_two_row_scales():
    # row n = 2^(n-3) * base: every row's gamma scales exactly and its codes equal the base row's
    base = synth.weights(1, 512, 0.02, 62).float().numpy()[0]
    W = np.stack([base * np.float32(2.0 ** (n - 3)) for n in range(8)]).astype(np.float32)
    Wp, g = oracle.pack_weights_rowwise(W)
    for n in range(8):
        assert g[n] == np.float32(g[3] * np.float32(2.0 ** (n - 3)))
    q, _ = oracle.unpack(Wp, 512)
    # eps = 1e-5 in d = gamma + eps shifts the boundaries by ~1e-5 / gamma: allow rare flips
    assert np.mean(q != q[3]) < 1e-3


def test_forward_rowwise_with_equal_gammas_is_forward():
    K, N, M = 256, 48, 3
    Wp, gamma = oracle.pack_weights(bf16_bits(synth.weights(N, K, 0.02, 63)))
    x = bf16_bits(synth.activations(M, K, seed=64, outliers=True))
    res = bf16_bits(synth.activations(M, N, seed=65, outliers=False))
    a = oracle.forward_rowwise(Wp, np.full(N, gamma, np.float32), x, residual=res)
    b = oracle.forward(Wp, gamma, x, residual=res)
    assert np.array_equal(a["acc"], b["acc"]) and np.array_equal(a["y"], b["y"])


def test_forward_rowwise_worked_2x4():
    # Hand-derived two-token forward over the per-row golden weights: the two rows
    # have different gammas and the two tokens different scales, so taking the
    # token's index for the row's gamma, or one gamma for every row, fails here.
    g = json.load(open(os.path.join(GOLDEN, "rowwise_2x4.json")))
    fw = g["forward"]
    Wp = np.array(g["packed"], np.uint8)
    gammas = np.array(g["gammas"], np.float32)
    x = bf16_bits(torch.tensor(fw["x"], dtype=torch.float32).to(torch.bfloat16))
    xq, s, xs = oracle.quant_act(x)
    assert xq.tolist() == fw["xq"] and s.tolist() == fw["s"] and xs.tolist() == fw["xsum"]
    # the dequantisation the variant defines, per output element
    y32 = np.array(fw["y32"], np.float32)
    for m in range(2):
        for n in range(2):
            assert np.float32(fw["acc"][m][n]) * (gammas[n] / s[m]) == y32[m, n]
    out = oracle.forward_rowwise(Wp, gammas, x)
    assert out["acc"].tolist() == fw["acc"]
    want = bf16_bits(torch.tensor(fw["y"], dtype=torch.float32).to(torch.bfloat16))
    assert np.array_equal(out["y"], want)
    assert np.array_equal(want, bf16_bits(torch.from_numpy(y32).to(torch.bfloat16)))
    res = bf16_bits(torch.tensor(fw["residual"], dtype=torch.float32).to(torch.bfloat16))
    out_r = oracle.forward_rowwise(Wp, gammas, x, residual=res)
    want_r = bf16_bits(torch.tensor(fw["y_residual"], dtype=torch.float32).to(torch.bfloat16))
    assert np.array_equal(out_r["y"], want_r)
    # neither the per-tensor path nor a transposed gamma choice reproduces it
    for wrong in (np.full(2, gammas[0], np.float32), gammas[::-1].copy()):
        assert not np.array_equal(oracle.forward_rowwise(Wp, wrong, x)["y"], want)


# ----------------------------------------------------------------------------- tensor-parallel pieces

@pytest.mark.parametrize("P", [1, 2, 3])
def test_ffn_tensor_parallel_pieces_compose_to_the_whole_layer(P):
    """Shards of the hidden width, combined with sums (fp64 statistics, int32
    accumulators) and maxima, give exactly the unsharded gammas, packed bytes, h,
    requantisation scale, accumulators and output. A slip such as dividing the
    sum of squares by the shard's width, a shard-local max, or a shard-local gamma
    breaks one of these equalities."""
    from bitlinear_w1_a8_02_b200 import tp
    d, f, M = 64, 200, 5
    Wg = bf16_bits(synth.weights(f, d, 0.02, 80))
    Wu = bf16_bits(synth.weights(f, d, 0.02, 81))
    Wd = bf16_bits(synth.weights(d, f, 0.02, 82))
    x = bf16_bits(synth.activations(M, d, seed=83, outliers=True))
    whole = [oracle.pack_weights(W) for W in (Wg, Wu, Wd)]
    ref = oracle.ffn_layer(whole[0][0], whole[0][1], whole[1][0], whole[1][1], whole[2][0], whole[2][1], x,
                           residual=x)
    bounds = [tp.shard_range(f, P, r, align=4) for r in range(P)]
    shards = []
    for (c0, c1) in bounds:
        parts = (Wg[c0:c1], Wu[c0:c1], np.ascontiguousarray(Wd[:, c0:c1]))
        shards.append(parts)
    packed = []
    for i, W in enumerate((Wg, Wu, Wd)):
        total = sum(oracle.absmean_sum(s[i]) for s in shards)
        packed.append([oracle.pack_weights_global(s[i], total, W.size) for s in shards])
        for r, (c0, c1) in enumerate(bounds):
            assert packed[i][r][1] == whole[i][1]
            want = whole[i][0][c0:c1] if i < 2 else whole[i][0][:, c0 // 4:c1 // 4]
            assert np.array_equal(packed[i][r][0], want)
    ups = [oracle.ffn_tp_up(packed[0][r][0], packed[0][r][1], packed[1][r][0], packed[1][r][1], x)
           for r in range(P)]
    assert np.array_equal(np.concatenate([u[0] for u in ups], axis=1), ref["h"])
    ss = np.zeros(M, np.float64)
    for u in ups:
        ss = ss + u[1]
    hmax = np.max(np.stack([u[2] for u in ups]), axis=0)
    acc = np.zeros((M, d), np.int64)
    s2 = None
    for r in range(P):
        a, s2r = oracle.ffn_tp_down(packed[2][r][0], ups[r][0], ss, hmax, f)
        acc += a
        assert s2 is None or np.array_equal(s2r, s2)
        s2 = s2r
    assert np.array_equal(s2, ref["s2"])
    assert np.array_equal(acc.astype(np.int32), ref["accd"])
    y = oracle.dequant(acc.astype(np.int32), packed[2][0][1], s2, residual=x)
    assert np.array_equal(y, ref["y"])


def test_pack_weights_global_keeps_the_eps():
    """Two one-row shards of the tensor of the eps example: mean |W| = 1/4 over the
    whole tensor, and w0 / (1/4 + 1e-5) < 0.5 gives code 0, where w0 / (1/4) =
    0.5 + 2^-18 would give 1. Codes [0, 1, 1, 1] are stored as q + 1 = [1, 2, 2, 2]
    at bits 0, 2, 4, 6: 1 + 2*4 + 2*16 + 2*64 = 169 (170 without the eps)."""
    row = [0.125 + 2.0 ** -20, 0.375 - 2.0 ** -20, 0.25, 0.25]
    shards = [np.array([row], np.float32), np.array([row], np.float32)]
    total = sum(oracle.absmean_sum(w) for w in shards)
    assert total == 2.0
    for w in shards:
        Wp, g = oracle.pack_weights_global(w, total, 8)
        assert g == np.float32(0.25)
        assert Wp.tolist() == [[169]]


def test_ffn_tensor_parallel_statistics_are_exact_sums():
    """A rank's subln statistics: ss is the fp64 sum of the exact squares of its h
    (each square of an fp32 value is exact in fp64), so it agrees with the
    correctly rounded sum to within the rounding of 200 fp64 additions; squares
    rounded to fp32 first would be off by ~1e-8 relative. hmax is max |h|."""
    d, f, M = 64, 200, 5
    Wg, gg = oracle.pack_weights(bf16_bits(synth.weights(f, d, 0.02, 80)))
    Wu, gu = oracle.pack_weights(bf16_bits(synth.weights(f, d, 0.02, 81)))
    x = bf16_bits(synth.activations(M, d, seed=83, outliers=True))
    h, ss, hmax = oracle.ffn_tp_up(Wg, gg, Wu, gu, x)
    assert np.count_nonzero(h) > M * f // 4
    for m in range(M):
        exact = math.fsum(float(v) ** 2 for v in h[m])
        assert abs(ss[m] - exact) <= 1e-12 * exact
        assert hmax[m] == np.abs(h[m]).max()


def test_ffn_tensor_parallel_requantisation_rounds_like_the_whole_layer():
    """The rank-local requantisation with the global statistics reproduces, code for
    code, the subln then per-token quantisation of the whole layer: hn = fl(h r),
    then rint(fl(hn s2)). h is drawn uniform in [-1, 1] (codes spread over the whole
    int8 range) and large enough that the other rounding order, rint(fl(h fl(r
    s2))), moves some code; the test checks that it does. The down weights are a
    row of +1 and a row of seeded ternary codes, so a moved code changes acc."""
    rng = np.random.default_rng(5)
    M, fl = 10, 262144
    h = rng.uniform(-1.0, 1.0, (M, fl)).astype(np.float32)
    # an all-zero token and one so small that max |h r| < 1e-5: both take the
    # scale floor, s2 = 127 / 1e-5, as the whole layer's quantisation does
    h[8] = 0.0
    h[9] *= np.float32(1e-9)
    codes = np.stack([np.ones(fl, np.int8), rng.integers(-1, 2, fl).astype(np.int8)])
    Wd = oracle.pack(codes)
    q2 = np.empty((M, fl), np.int8)
    s2 = np.empty(M, np.float32)
    moved = 0
    for m in range(M):
        r, hn = oracle.subln_rms(h[m])
        xq, s, _ = oracle.quant_act(hn[None, :])
        q2[m], s2[m] = xq[0], s[0]
        other = np.clip(np.rint(h[m] * np.float32(r * s[0])), -128, 127).astype(np.int8)
        moved += int(np.count_nonzero(other != q2[m]))
    assert moved > 0
    # ss in the order the whole layer sums it (sequential fp64 over j), hmax exact
    ss = np.cumsum(h.astype(np.float64) ** 2, axis=1)[:, -1]
    hmax = np.abs(h).max(axis=1)
    acc, s2_tp = oracle.ffn_tp_down(Wd, h, ss, hmax, fl)
    assert s2[8] == s2[9] == np.float32(127.0) / np.float32(1e-5)
    assert np.array_equal(s2_tp, s2)
    assert np.array_equal(acc, (q2.astype(np.int64) @ codes.T.astype(np.int64)).astype(np.int32))

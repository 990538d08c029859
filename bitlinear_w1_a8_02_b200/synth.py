"""Seeded synthetic inputs shaped like a 2B-parameter ternary model.

This module holds no arithmetic of the method: it only draws random tensors.
Both the CUDA path's tests/benchmark and the CPU oracle are fed from here.

Recipe (torch's counter-based Philox generator on CUDA, its Mersenne-Twister
generator on CPU; values for a seed differ between the two devices, so one test
or benchmark run draws on one device and hands the same bytes to both sides):
  * weights W [N, K]: N(0, sigma^2) drawn in fp32, then rounded to bf16 (RN), or
    kept fp32 for the small fp32-weight case;
  * activations x [M, K]: N(0, 1) in fp32; floor(0.01 * K) outlier channels,
    picked by a seeded permutation and shared by every token, are multiplied by
    20; then rounded to bf16.
"""
from __future__ import annotations

import torch

SIGMA_2B = 0.02
SIGMA_100B = 0.01
OUTLIER_FRACTION = 0.01
OUTLIER_SCALE = 20.0

# The five workloads the library is measured and checked on.
CONFIGS = {
    "single": dict(M=[1], shapes=[(256, 512)], sigma=SIGMA_2B, w_dtype="fp32", outliers=False),
    "decode_2b": dict(M=[1], shapes=[(2560, 2560), (2560, 640), (2560, 6912), (6912, 2560)],
                      sigma=SIGMA_2B, w_dtype="bf16", outliers=True, copies=30),
    "batched_2b": dict(M=[4, 8, 16, 512, 2048, 4096], shapes=[(2560, 6912), (6912, 2560)],
                       sigma=SIGMA_2B, w_dtype="bf16", outliers=True),
    "ffn_2b": dict(M=[1, 512], d=2560, f=6912, layers=30, sigma=SIGMA_2B, w_dtype="bf16",
                   outliers=False),
    "stress_100b": dict(M=[1, 16, 2048], shapes=[(8192, 28672), (28672, 8192)],
                        sigma=SIGMA_100B, w_dtype="bf16", outliers=True),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(N: int, K: int, sigma: float, seed: int, dtype: str = "bf16",
            device="cpu") -> torch.Tensor:
    """W [N, K] ~ N(0, sigma^2), as bf16 (default) or fp32."""
    g = _gen(seed, device)
    w = torch.randn((N, K), generator=g, dtype=torch.float32, device=device)
    w.mul_(sigma)
    return w if dtype == "fp32" else w.to(torch.bfloat16)


def outlier_channels(K: int, seed: int, device="cpu") -> torch.Tensor:
    n = int(OUTLIER_FRACTION * K)
    g = _gen(seed + 0x5EED, "cpu")
    return torch.randperm(K, generator=g)[:n].to(device)


def activations(M: int, K: int, seed: int, outliers: bool = True, device="cpu") -> torch.Tensor:
    """x [M, K] bf16 ~ N(0, 1), with 1% of channels scaled by 20 when asked."""
    g = _gen(seed, device)
    x = torch.randn((M, K), generator=g, dtype=torch.float32, device=device)
    if outliers and M > 0:
        ch = outlier_channels(K, seed, device)
        x[:, ch] *= OUTLIER_SCALE
    return x.to(torch.bfloat16)


def weight_seed(shape_index: int, copy: int) -> int:
    """Seed of copy ``copy`` (one per layer) of the shape ``shape_index``."""
    return 1000 * (shape_index + 1) + copy


def ffn_layer_seeds(layer: int):
    """Seeds of the gate, up and down weights of FFN layer ``layer``."""
    return 3 * layer, 3 * layer + 1, 3 * layer + 2

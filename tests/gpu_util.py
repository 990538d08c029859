"""Shared helpers of the GPU parity tests: tensor <-> numpy bit patterns and the
comparison rules (bit-exact integers; bf16 within 2^-8 relative, 1e-3 absolute
near zero, and in this library also bit-exact)."""
import numpy as np
import torch

import oracle

REL_TOL = 2.0 ** -8
ABS_TOL = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def np_(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def assert_bf16_close(got_bits: np.ndarray, ref_bits: np.ndarray, what: str = "y"):
    """The published bar: |got - ref| <= 2^-8 |ref|, or <= 1e-3 where |ref| is
    below 1e-3 of the tensor's RMS."""
    g = oracle.bf16_to_f32(got_bits).astype(np.float64)
    r = oracle.bf16_to_f32(ref_bits).astype(np.float64)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    near0 = np.abs(r) < 1e-3 * rms
    err = np.abs(g - r)
    ok = np.where(near0, err <= ABS_TOL, err <= REL_TOL * np.abs(r))
    bad = np.argwhere(~ok)
    assert bad.size == 0, f"{what}: {len(bad)} of {ok.size} outside tolerance, first at {bad[:4].tolist()}"


def assert_bf16_exact(got_bits: np.ndarray, ref_bits: np.ndarray, what: str = "y"):
    diff = np.argwhere(got_bits != ref_bits)
    assert diff.size == 0, f"{what}: {len(diff)} of {got_bits.size} bf16 values differ, first at {diff[:4].tolist()}"


def sample_indices(n: int, k: int, seed: int) -> np.ndarray:
    """k sorted distinct indices of range(n), always including the first and last."""
    if n <= k:
        return np.arange(n)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, n - 1), size=k - 2, replace=False)
    return np.sort(np.concatenate([[0, n - 1], mid]))

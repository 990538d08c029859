"""Tensor-parallel FFN sub-layer over torch.distributed ranks (one GPU each).

The pages give no distributed detail (paper card "BitNet b1.58 2B4T Technical
Report", "Limits"); this is the library's split of the FFN sub-layer of
bitlinear_ffn over P ranks. Rank r owns the hidden columns [c0, c1) of f: those
rows of the gate and up weights and those columns of the down weight. Every
rank holds the whole x and residual. Exchanges (NCCL over NVLink on GPUs):

  * at pack time, the fp64 sum of |W| of each weight (sum over ranks), so every
    shard is ternarised with the gamma of the whole tensor (per-tensor absmean,
    paper card "Method Adaptation");
  * per layer, the per-token subln statistics after gate/up: sum h^2 (fp64, sum)
    and max |h| (fp32, max), so the RMSNorm factor and the requantisation scale
    are those of the whole row;
  * the down projection's int32 accumulators (sum; exact in any order), then the
    dequantisation with the residual on every rank.

The per-rank compute is an object with five methods (absmean_sum, pack_global,
ffn_up, ffn_down, ffn_finish); CudaRankOps runs them in the library's kernels.
This module holds only the orchestration: it computes nothing itself.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist

from . import binding as _b


def shard_range(f: int, world: int, rank: int, align: int = 256):
    """Hidden columns [c0, c1) owned by `rank`: boundaries on multiples of `align`
    (256 keeps every shard on the streamed kernels), as even as possible; the
    last rank also takes the remainder below `align`."""
    units = f // align
    if units < world:
        raise ValueError(f"f = {f} gives fewer than {world} shards of {align} columns")

    def bound(r):
        return f if r == world else align * int(units * r / world + 0.5)
    return bound(rank), bound(rank + 1)


class CudaRankOps:
    """Per-rank compute in the library's CUDA kernels (through the C ABI)."""

    def absmean_sum(self, W):
        return _b.absmean_sum(W)

    def pack_global(self, W, total_sum, total_count):
        return _b.pack_weights_global(W, total_sum, total_count)

    def ffn_up(self, Wg, gg, Wu, gu, x):
        return _b.ffn_tp_up(Wg, gg, Wu, gu, x)

    def ffn_down(self, Wd, h, ss_all, hmax_all, f_total):
        return _b.ffn_tp_down(Wd, h, ss_all, hmax_all, f_total)

    def ffn_finish(self, acc, gd, s2, residual):
        return _b.ffn_tp_finish(acc, gd, s2, residual)


@dataclass
class FfnShard:
    """A rank's packed share of one FFN sub-layer."""
    Wg: torch.Tensor   # [f_local, d/4] gate rows
    gg: torch.Tensor   # [1] gamma of the whole gate weight
    Wu: torch.Tensor   # [f_local, d/4] up rows
    gu: torch.Tensor
    Wd: torch.Tensor   # [d, f_local/4] down columns
    gd: torch.Tensor
    f_total: int
    c0: int
    c1: int


def _distributed(group) -> bool:
    """True when a process group exists (one rank included: the exchanges then run
    as one-rank collectives, which change nothing)."""
    return dist.is_available() and dist.is_initialized()


def _all_reduce(t: torch.Tensor, op, group):
    if _distributed(group):
        dist.all_reduce(t, op=op, group=group)
    return t


def pack_ffn_shard(Wg_rows, Wu_rows, Wd_cols, f_total: int, c0: int, c1: int, group=None,
                   ops=None) -> FfnShard:
    """Pack this rank's shard: Wg_rows, Wu_rows [f_local, d] and Wd_cols [d, f_local]
    (bf16 or fp32) with the gammas of the whole tensors (one fp64 all-reduce each)."""
    ops = CudaRankOps() if ops is None else ops
    packed = []
    for W in (Wg_rows, Wu_rows, Wd_cols):
        total = ops.absmean_sum(W)
        _all_reduce(total, dist.ReduceOp.SUM, group)
        count = W.shape[0] * W.shape[1] * f_total // (c1 - c0)
        packed.append(ops.pack_global(W, total, count))
    (Wg, gg), (Wu, gu), (Wd, gd) = packed
    return FfnShard(Wg, gg, Wu, gu, Wd, gd, f_total, c0, c1)


def ffn_tp(shard: FfnShard, x: torch.Tensor, residual: Optional[torch.Tensor] = None, group=None, ops=None):
    """One FFN sub-layer on this rank's shard; every rank returns the whole y [M, d]."""
    ops = CudaRankOps() if ops is None else ops
    h, ss, hmax = ops.ffn_up(shard.Wg, shard.gg, shard.Wu, shard.gu, x)
    _all_reduce(ss, dist.ReduceOp.SUM, group)
    _all_reduce(hmax, dist.ReduceOp.MAX, group)
    acc, s2 = ops.ffn_down(shard.Wd, h, ss, hmax, shard.f_total)
    _all_reduce(acc, dist.ReduceOp.SUM, group)
    return ops.ffn_finish(acc, shard.gd, s2, residual)

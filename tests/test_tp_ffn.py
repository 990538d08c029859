"""The tensor-parallel FFN sub-layer (bitlinear_w1_a8_02_b200.tp).

CPU: two gloo ranks run the library's orchestration (pack_ffn_shard, ffn_tp) with
rank-local compute from the oracle's tensor-parallel pieces, and must reproduce
the oracle's unsharded FFN layer bit for bit; this checks the split and the
collectives (fp64 sums, fp32 maxima, exact int32 sums).

GPU (one device): the library's kernels for each shard of P = 2 and 4 ranks,
the exchanges done as device sums and maxima, against the oracle's pieces and
the unsharded layer; and ffn_tp itself over a one-rank NCCL process group.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bitlinear_w1_a8_02_b200 import synth, tp


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleRankOps:
    """Rank-local compute from the oracle's tensor-parallel pieces (CPU tensors)."""

    def absmean_sum(self, W):
        return torch.tensor([oracle.absmean_sum(_bits(W))], dtype=torch.float64)

    def pack_global(self, W, total_sum, total_count):
        Wp, g = oracle.pack_weights_global(_bits(W), float(total_sum[0]), int(total_count))
        return torch.from_numpy(Wp), torch.tensor([g], dtype=torch.float32)

    def ffn_up(self, Wg, gg, Wu, gu, x):
        h, ss, hmax = oracle.ffn_tp_up(Wg.numpy(), float(gg[0]), Wu.numpy(), float(gu[0]), _bits(x))
        return torch.from_numpy(h), torch.from_numpy(ss), torch.from_numpy(hmax)

    def ffn_down(self, Wd, h, ss_all, hmax_all, f_total):
        acc, s2 = oracle.ffn_tp_down(Wd.numpy(), h.numpy(), ss_all.numpy(), hmax_all.numpy(), f_total)
        return torch.from_numpy(acc), torch.from_numpy(s2)

    def ffn_finish(self, acc, gd, s2, residual):
        y = oracle.dequant(acc.numpy(), float(gd[0]), s2.numpy(), residual=None if residual is None else _bits(residual))
        return torch.from_numpy(y.view(np.int16)).view(torch.bfloat16)


D, F, M = 64, 200, 5


def _layer_weights():
    return (synth.weights(F, D, 0.02, 90), synth.weights(F, D, 0.02, 91), synth.weights(D, F, 0.02, 92))


def _gloo_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Wg, Wu, Wd = _layer_weights()
        c0, c1 = tp.shard_range(F, world, rank, align=4)
        ops = OracleRankOps()
        shard = tp.pack_ffn_shard(Wg[c0:c1].contiguous(), Wu[c0:c1].contiguous(), Wd[:, c0:c1].contiguous(), F,
                                  c0, c1, ops=ops)
        h = synth.activations(M, D, seed=93, outliers=True)
        for _ in range(2):  # two layers in a row on the same shard
            h = tp.ffn_tp(shard, h, residual=h, ops=ops)
        out[rank] = _bits(h).astype(np.int64).tolist()
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_reproduce_the_unsharded_layer():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:  # no fork: CUDA may be initialised in this process
        out = mgr.dict()
        mp.spawn(_gloo_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        got = [np.array(out[r], np.uint16) for r in range(world)]
    Wg, Wu, Wd = _layer_weights()
    P = [oracle.pack_weights(_bits(W)) for W in (Wg, Wu, Wd)]
    h = _bits(synth.activations(M, D, seed=93, outliers=True))
    for _ in range(2):
        h = oracle.ffn_layer(P[0][0], P[0][1], P[1][0], P[1][1], P[2][0], P[2][1], h, residual=h)["y"]
    for g in got:
        assert np.array_equal(g, h)


# ----------------------------------------------------------------------------- GPU

def _emulated(d, f, Mt, world, dev, seed):
    """P ranks on one GPU: each shard through the library's kernels; the
    exchanges as device sums and maxima. Checked against the oracle's pieces and
    the unsharded oracle layer."""
    import bitlinear_w1_a8_02_b200 as bl
    Ws = [synth.weights(f, d, 0.02, seed), synth.weights(f, d, 0.02, seed + 1), synth.weights(d, f, 0.02, seed + 2)]
    x = synth.activations(Mt, d, seed=seed + 3, outliers=False)
    bounds = [tp.shard_range(f, world, r) for r in range(world)]
    shards = [(W_g[c0:c1], W_u[c0:c1], W_d[:, c0:c1]) for (c0, c1) in bounds for (W_g, W_u, W_d) in [Ws]]
    packed = []  # per rank: (Wg, gg, Wu, gu, Wd, gd) on the device
    for i in range(3):
        parts = [s[i].contiguous().to(dev) for s in shards]
        total = sum(bl.absmean_sum(p) for p in parts)
        packed.append([bl.pack_weights_global(p, total, Ws[i].numel()) for p in parts])
    whole = [oracle.pack_weights(_bits(W)) for W in Ws]
    for i in range(3):
        for r, (c0, c1) in enumerate(bounds):
            assert np.float32(packed[i][r][1].cpu()[0]) == whole[i][1]
            want = whole[i][0][c0:c1] if i < 2 else whole[i][0][:, c0 // 4:c1 // 4]
            assert np.array_equal(packed[i][r][0].cpu().numpy(), want)
    xd = x.to(dev)
    ups = [bl.ffn_tp_up(packed[0][r][0], packed[0][r][1], packed[1][r][0], packed[1][r][1], xd) for r in range(world)]
    for r in range(world):
        h_ref, ss_ref, mx_ref = oracle.ffn_tp_up(packed[0][r][0].cpu().numpy(), whole[0][1],
                                                 packed[1][r][0].cpu().numpy(), whole[1][1], _bits(x))
        assert np.array_equal(ups[r][0].cpu().numpy(), h_ref)
        assert np.array_equal(ups[r][2].cpu().numpy(), mx_ref)
        assert np.allclose(ups[r][1].cpu().numpy(), ss_ref, rtol=1e-12, atol=0)
    ss = sum(u[1] for u in ups)
    hmax = torch.stack([u[2] for u in ups]).amax(dim=0)
    downs = [bl.ffn_tp_down(packed[2][r][0], ups[r][0], ss, hmax, f) for r in range(world)]
    acc = sum(a for a, _ in downs)
    y = bl.ffn_tp_finish(acc, packed[2][0][1], downs[0][1], residual=xd)
    ref = oracle.ffn_layer(whole[0][0], whole[0][1], whole[1][0], whole[1][1], whole[2][0], whole[2][1], _bits(x),
                           residual=_bits(x))
    assert np.array_equal(acc.cpu().numpy(), ref["accd"])
    assert np.array_equal(downs[0][1].cpu().numpy(), ref["s2"])
    assert np.array_equal(_bits(y), ref["y"])
    assert bl.get_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("Mt", [1, 5, 300])
def test_emulated_ranks_on_one_gpu(cuda_device, world, Mt):
    _emulated(2560, 6912, Mt, world, cuda_device, seed=900 + world + Mt)


@pytest.mark.gpu
def test_ffn_tp_over_one_rank_nccl(cuda_device):
    """ffn_tp's NCCL path with a one-rank group equals the library's bitlinear_ffn."""
    import bitlinear_w1_a8_02_b200 as bl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=cuda_device)
    try:
        d, f, Mt = 2560, 6912, 4
        Wg, Wu, Wd = (synth.weights(f, d, 0.02, 950).to(cuda_device), synth.weights(f, d, 0.02, 951).to(cuda_device),
                      synth.weights(d, f, 0.02, 952).to(cuda_device))
        shard = tp.pack_ffn_shard(Wg, Wu, Wd, f, 0, f)
        x = synth.activations(Mt, d, seed=953, outliers=False).to(cuda_device)
        y = tp.ffn_tp(shard, x, residual=x)
        P = [bl.pack_weights(W) for W in (Wg, Wu, Wd)]
        y_ref = bl.ffn(P[0][0], P[0][1], P[1][0], P[1][1], P[2][0], P[2][1], x, residual=x)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    finally:
        dist.destroy_process_group()

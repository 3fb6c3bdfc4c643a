"""Data-parallel path on CPU: two gloo ranks, each with its own token shard.

Each rank computes its shard's dA, dB with the oracle (the CUDA path needs a
GPU), writes them into a GradBucket and sums them with one all-reduce; the sum
must equal the full-batch oracle gradients (the gradients are sums over
tokens, so splitting the batch and adding the parts changes only the rounding
order).  Also checks that the shards cover every token exactly once.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_pack_b200.dp import GradBucket, shard_tokens


def test_shards_cover_tokens_once():
    for M in (0, 1, 7, 64, 4097):
        for world in (1, 2, 3, 8):
            seen = np.zeros(M, dtype=int)
            for rank in range(world):
                sl = shard_tokens(M, world, rank)
                seen[sl] += 1
            assert (seen == 1).all(), (M, world)
    with pytest.raises(ValueError):
        shard_tokens(8, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    from inputs import synthetic as S
    from tests._gpu_util import OracleWeight
    M, K, N, r = 37, 128, 192, 8
    lin = S.random_case(4242, M, K, N, r)
    lin.dY = S.normal(4243, M, 4, (M, N), 1.0)
    return lin, OracleWeight(lin.W, True).w_hat, 32.0 / r


def _worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle.linear import lora_backward
        lin, w_hat, c = _case()
        M, K = lin.X.shape
        N, r = lin.dY.shape[1], lin.A.shape[1]
        sl = shard_tokens(M, world, rank)
        _, dA, dB = lora_backward(lin.dY[sl], lin.X[sl], w_hat, lin.A, lin.B, c)
        g = GradBucket(K, N, r, "cpu")
        g.dA.copy_(torch.from_numpy(dA))
        g.dB.copy_(torch.from_numpy(dB))
        g.all_reduce()
        if rank == 0:
            np.savez(out_path, dA=g.dA.numpy(), dB=g.dB.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_gradient_sum(tmp_path):
    from oracle.linear import lora_backward
    out = str(tmp_path / "dp.npz")
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    lin, w_hat, c = _case()
    _, dA, dB = lora_backward(lin.dY, lin.X, w_hat, lin.A, lin.B, c)
    got = np.load(out)
    # fp32 bucket: the per-shard fp64 sums are rounded once each, then added
    for ref, g in ((dA, got["dA"]), (dB, got["dB"])):
        err = np.linalg.norm(g - ref) / np.linalg.norm(ref)
        assert err < 1e-6, err

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


# ---------------------------------------------------------------------------
# Sharded quantization across two gloo ranks.  The device phases are replaced
# by stand-ins written with the oracle (the CUDA path needs a GPU): what this
# checks is the host orchestration of dp.quantize_data_parallel (block ranges
# in whole groups, one integer all-reduce of the exponent bins, the all-gather
# of every range) against the oracle's single-rank quantization, bit for bit.
# ---------------------------------------------------------------------------
class _CpuState:
    def __init__(self, shape, dq, device, codebook=0):
        n = int(np.prod(shape))
        n1 = -(-n // 64)
        self.packed = torch.zeros((n + 1) // 2, dtype=torch.uint8)
        self.dq = dq
        if dq:
            self.code8 = torch.zeros(n1, dtype=torch.uint8)
            self.s2 = torch.zeros(-(-n1 // 256), dtype=torch.float32)
            self.offset = torch.zeros(1, dtype=torch.float32)
        else:
            self.absmax = torch.zeros(n1, dtype=torch.float32)


def _bins_of(scales):
    """The exponent bins the encoder keeps: per biased exponent E (1 for
    subnormals) the sum of the 24-bit integer significands."""
    u = np.asarray(scales, np.float32).view(np.uint32).astype(np.int64)
    E = (u >> 23) & 0xFF
    mant = (u & 0x7FFFFF) | np.where(E > 0, 0x800000, 0)
    bins = np.zeros(256, dtype=np.int64)
    np.add.at(bins, np.maximum(E, 1), mant)
    return bins


def _fake_begin(W_shard, w, b0, b1, workspace=None):
    from oracle import nf4
    if b1 == b0:
        if workspace is not None:
            workspace[:2048].zero_()
        return
    codes, absmax = nf4.quantize_nf4(W_shard.numpy().astype(np.float32))
    payload, _ = nf4.pack_codes(codes)
    w.packed[b0 * 32: b0 * 32 + payload.size] = torch.from_numpy(payload)
    if not w.dq:
        w.absmax[b0:b1] = torch.from_numpy(absmax)
        return
    workspace[:2048].view(torch.int64).copy_(torch.from_numpy(_bins_of(absmax)))
    workspace[2304: 2304 + 4 * (b1 - b0)].view(torch.float32).copy_(torch.from_numpy(absmax))


def _fake_end(w, b0, b1, workspace=None):
    from fractions import Fraction

    from oracle import nf4
    bins = workspace[:2048].view(torch.int64).numpy()
    n1 = w.code8.numel()
    total = sum(Fraction(int(v)) * Fraction(2) ** (k - 150) for k, v in enumerate(bins) if v)
    mean = total / n1
    offset = nf4._round_rational_to_f32(mean.numerator, mean.denominator)
    w.offset[0] = float(offset)
    if b1 > b0:
        scales = workspace[2304: 2304 + 4 * (b1 - b0)].view(torch.float32).numpy()
        code8, s2, _ = nf4.double_quantize_centred(scales, offset)
        w.code8[b0:b1] = torch.from_numpy(code8)
        w.s2[b0 // 256: b0 // 256 + s2.size] = torch.from_numpy(s2)


def _quant_worker(rank, world, port, out_path, shape, dq):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from bit_nf4_quantized_pack_b200.dp import quantize_data_parallel
        W = _quant_input(shape)
        w = quantize_data_parallel(torch.from_numpy(W), dq, begin=_fake_begin, end=_fake_end,
                                   new_weight=_CpuState)
        out = {"packed": w.packed.numpy()}
        if dq:
            out.update(code8=w.code8.numpy(), s2=w.s2.numpy(), offset=w.offset.numpy())
        else:
            out.update(absmax=w.absmax.numpy())
        np.savez(out_path + f".{rank}.npz", **out)
    finally:
        dist.destroy_process_group()


def _quant_input(shape):
    from inputs import synthetic as S
    W = S.normal(77, 5, 0, shape, 0.02)
    W.reshape(-1)[640:704] = 0.0                     # an all-zero block
    return W


@pytest.mark.parametrize("shape,dq", [((96, 700), True), ((40, 2048), True), ((33, 64), False)])
def test_two_rank_sharded_quantize_matches_single_rank_oracle(tmp_path, shape, dq):
    from oracle import nf4
    out = str(tmp_path / "q")
    mp.start_processes(_quant_worker, args=(2, _free_port(), out, shape, dq), nprocs=2, join=True,
                       start_method="spawn")
    W = _quant_input(shape)
    codes, absmax = nf4.quantize_nf4(W.ravel())
    payload, _ = nf4.pack_codes(codes)
    for rank in range(2):
        got = np.load(out + f".{rank}.npz")
        assert np.array_equal(got["packed"], payload)
        if dq:
            code8, s2, off = nf4.double_quantize(absmax)
            assert np.array_equal(got["code8"], code8)
            assert np.array_equal(got["s2"].view(np.uint32), s2.view(np.uint32))
            assert got["offset"].view(np.uint32)[0] == np.float32(off).view(np.uint32)
        else:
            assert np.array_equal(got["absmax"].view(np.uint32), absmax.view(np.uint32))


def test_shard_blocks_cover_whole_groups():
    from bit_nf4_quantized_pack_b200.dp import shard_blocks
    for n1 in (1, 255, 256, 257, 4096, 70000):
        for world in (1, 2, 3, 8):
            seen = np.zeros(n1, dtype=int)
            for rank in range(world):
                b0, b1 = shard_blocks(n1, world, rank)
                assert b0 == b1 or (b0 % 256 == 0 and (b1 % 256 == 0 or b1 == n1))
                seen[b0:b1] += 1
            assert (seen == 1).all(), (n1, world)

"""Data-parallel plumbing for the frozen-base LoRA layer.

Every rank holds the same frozen NF4 weight (quantized from the same bf16 W)
and the same adapter A, B, and runs the forward and backward on its own
tokens.  The frozen base gets no parameter update, only the adapter does (the
page "QLoRA：冻结的 4-bit 权重怎样参与一次微调", §冻结权重为什么仍然需要输入梯度),
so the one exchange of the step is the sum of dA and dB over ranks.  Both are small
(K·r and r·N fp32), so they travel as ONE all-reduce of a flat bucket: one
collective launch per step instead of two.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["shard_tokens", "GradBucket", "shard_blocks", "quantize_data_parallel"]

BLOCK = 64          # elements per first-level block
GROUP = 256         # first-level blocks per double-quantization group


def shard_tokens(M: int, world: int, rank: int) -> slice:
    """Rows [start, stop) of a global batch of M tokens owned by `rank`: the
    first M % world ranks take one extra row, so every token is owned once."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


class GradBucket:
    """dA (K x r) and dB (r x N) as views of one contiguous fp32 buffer, so the
    backward writes them in place and one all-reduce sums both."""

    def __init__(self, K: int, N: int, r: int, device) -> None:
        self.buf = torch.empty(K * r + r * N, dtype=torch.float32, device=device)
        self.dA = self.buf[: K * r].view(K, r)
        self.dB = self.buf[K * r:].view(r, N)

    def all_reduce(self, group=None) -> None:
        """Sum dA and dB over the ranks of `group` (in place)."""
        if dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.buf, op=dist.ReduceOp.SUM, group=group)


def shard_blocks(n1: int, world: int, rank: int, group_blocks: int = GROUP) -> tuple:
    """Blocks [b0, b1) of n1 that `rank` quantizes: whole groups of
    `group_blocks` blocks (so that each rank double-quantizes whole groups),
    the first ngroups % world ranks taking one group more; ranges may be
    empty when there are fewer groups than ranks."""
    if world < 1 or not 0 <= rank < world or n1 < 0 or group_blocks < 1:
        raise ValueError("bad shard request")
    ngroups = -(-n1 // group_blocks)
    base, extra = divmod(ngroups, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    return min(g0 * group_blocks, n1), min(g1 * group_blocks, n1)


def _gather_ranges(t: torch.Tensor, ranges, rank: int, group) -> None:
    """Every rank owns t[start:stop] of its entry in `ranges`; afterwards every
    rank holds every piece (one all-gather of equal-sized, padded pieces)."""
    width = max(stop - start for start, stop in ranges)
    if width == 0:
        return
    start, stop = ranges[rank]
    piece = torch.zeros(width, dtype=t.dtype, device=t.device)
    piece[: stop - start] = t[start:stop]
    outs = [torch.empty_like(piece) for _ in ranges]
    dist.all_gather(outs, piece, group=group)
    for (a, b), o in zip(ranges, outs):
        t[a:b] = o[: b - a]


def quantize_data_parallel(W: torch.Tensor, double_quant: bool = True, *, group=None,
                           codebook: str = "nf4", begin=None, end=None, new_weight=None):
    """Quantize the frozen weight once across the ranks of `group`, each rank
    encoding 1/world of the 64-blocks, and return the full quantized state on
    every rank, bit-identical to a single-device quantize of W.

    The exchange is one all-reduce of the 256 exponent bins of the first-level
    scales (64-bit integer sums, so the double quantization's exact mean is
    the same on every rank) and one all-gather of each rank's packed bytes and
    scale codes (page "SFT（四）：QLoRA的4-bit量化与LoRA微调原理", §26.1: the
    frozen base is replicated on every device of the data-parallel batch).
    `begin`, `end` and `new_weight` default to the library's entry points;
    another implementation with the same contract may be passed instead.
    """
    from . import NF4Weight, quantize_shard_begin, quantize_shard_end, shard_workspace_size
    begin = begin or quantize_shard_begin
    end = end or quantize_shard_end
    cb = 1 if codebook == "int4" else 0
    if cb:
        double_quant = False
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    numel = W.numel()
    n1 = -(-numel // BLOCK)
    ranges = [shard_blocks(n1, world, rr) for rr in range(world)]
    b0, b1 = ranges[rank]
    w = (new_weight or NF4Weight.empty)(tuple(W.shape), double_quant, W.device, codebook=cb)
    flat = W.reshape(-1)
    ws = None
    if double_quant:
        ws = torch.empty(max(256, shard_workspace_size(numel, b0, b1, True)), dtype=torch.uint8,
                         device=W.device)
    begin(flat[b0 * BLOCK: min(b1 * BLOCK, numel)], w, b0, b1, workspace=ws)
    if double_quant:
        bins = ws[:2048].view(torch.int64)       # 256 sums, each below 2^63
        if world > 1:
            dist.all_reduce(bins, op=dist.ReduceOp.SUM, group=group)
        end(w, b0, b1, workspace=ws)
    if world > 1:
        nbytes = (numel + 1) // 2
        _gather_ranges(w.packed, [(a * BLOCK // 2, min(b * BLOCK // 2, nbytes)) for a, b in ranges],
                       rank, group)
        if double_quant:
            _gather_ranges(w.code8, ranges, rank, group)
            _gather_ranges(w.s2, [(a // GROUP, -(-b // GROUP)) for a, b in ranges], rank, group)
        else:
            _gather_ranges(w.absmax, ranges, rank, group)
    return w

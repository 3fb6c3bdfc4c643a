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

__all__ = ["shard_tokens", "GradBucket"]


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

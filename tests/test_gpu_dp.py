"""Data parallelism through the CUDA library, on one GPU (the pool gives one
GPU per call, so the ranks run one after another on it; no kernel waits on
another rank's).

* Sharded quantization: each emulated rank encodes its range of 64-blocks
  with qlora_nf4_quantize_shard_begin, the exponent bins are summed over the
  ranks (the all-reduce), qlora_nf4_quantize_shard_end forms the offset and the
  scale codes of each range; the assembled state is bit-identical to one
  qlora_nf4_quantize of the whole weight.
* Token shards: each rank's backward on its tokens, dA and dB summed in a
  GradBucket, against the full-batch oracle gradients.
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_pack_b200.dp import GradBucket, shard_blocks, shard_tokens
from inputs import synthetic as S
from oracle.linear import lora_adapter_grads
from tests._gpu_util import assert_close, to_dev, to_np

pytestmark = pytest.mark.gpu


def _q():
    import bit_nf4_quantized_pack_b200 as q
    return q


@pytest.mark.parametrize("K,N,world,dq", [(1024, 1088, 2, True), (2048, 4160, 3, True),
                                          (640, 576, 2, False), (16, 640, 3, True)])
def test_sharded_quantize_is_bit_identical(K, N, world, dq):
    q = _q()
    lin = S.random_case(700 + K + N + world, 4, K, N, 8)
    W = to_dev(lin.W)
    W[1, 64:128] = 0                                  # an all-zero block
    ref = q.quantize(W, double_quant=dq)
    numel = K * N
    n1 = -(-numel // 64)
    w = q.NF4Weight.empty((K, N), dq, W.device)
    flat = W.reshape(-1)
    ranges = [shard_blocks(n1, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n1
    wss = []
    for b0, b1 in ranges:
        ws = torch.empty(max(256, q.shard_workspace_size(numel, b0, b1, dq)), dtype=torch.uint8,
                         device=W.device)
        q.quantize_shard_begin(flat[b0 * 64: min(b1 * 64, numel)], w, b0, b1, workspace=ws)
        wss.append(ws)
    if dq:
        total = sum(ws[:2048].view(torch.int64) for ws in wss)   # the all-reduce
        for (b0, b1), ws in zip(ranges, wss):
            ws[:2048].view(torch.int64).copy_(total)
            q.quantize_shard_end(w, b0, b1, workspace=ws)
    assert torch.equal(w.packed, ref.packed)
    if dq:
        assert torch.equal(w.code8, ref.code8)
        assert torch.equal(w.s2.view(torch.int32), ref.s2.view(torch.int32))
        assert torch.equal(w.offset.view(torch.int32), ref.offset.view(torch.int32))
    else:
        assert torch.equal(w.absmax.view(torch.int32), ref.absmax.view(torch.int32))


def test_sharded_quantize_rejects_ranges_that_split_a_group():
    q = _q()
    W = torch.zeros((64, 1024), dtype=torch.bfloat16, device="cuda")
    w = q.NF4Weight.empty((64, 1024), True, W.device)
    ws = torch.empty(1 << 16, dtype=torch.uint8, device=W.device)
    with pytest.raises(q.QLoRAError):
        q.quantize_shard_begin(W.reshape(-1)[64 * 128:], w, 128, 1024, workspace=ws)


def test_token_shards_sum_to_full_batch_gradients():
    q = _q()
    M, K, N, r, world = 600, 512, 768, 16, 3
    lin = S.random_case(4321, M, K, N, r)
    lin.dY = S.normal(4322, M, 4, (M, N), 1.0)
    c = 2.0
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    At, Bt = to_dev(lin.A), to_dev(lin.B)
    total = GradBucket(K, N, r, "cuda")
    total.buf.zero_()
    for rank in range(world):
        sl = shard_tokens(M, world, rank)
        Xs, Gs = to_dev(lin.X[sl]), to_dev(lin.dY[sl])
        _, Zc = q.linear_forward(Xs, wq, At, Bt, c)
        g = GradBucket(K, N, r, "cuda")
        q.linear_backward(Gs, Xs, Zc, wq, At, Bt, c, dA=g.dA, dB=g.dB)
        total.buf += g.buf                            # the all-reduce of the bucket
    _, dAr, dBr = lora_adapter_grads(lin.dY, lin.X, lin.A, lin.B, c)
    assert_close("dA", to_np(total.dA), dAr)
    assert_close("dB", to_np(total.dB), dBr)

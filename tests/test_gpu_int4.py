"""The uniform signed INT4 codebook through the library's kernels, against
the oracle's INT4 storage format (``oracle/int4.py``).

Bit-exact: codes, stored scales, padding and the decoded bf16 weights.
Forward, backward, GEMV and merge: relative Frobenius <= 5e-3 against the
fp64 oracle on the oracle's decoded INT4 weight (merge: one bf16 ulp).
"""
import numpy as np
import pytest
import torch

from inputs import synthetic as S
from oracle.int4 import int4_dequantize, int4_quantize
from oracle.linear import lora_backward, lora_forward
from oracle.merge import merge_bf16, merge_exact
from tests._gpu_util import rel_fro, to_dev, to_np

pytestmark = pytest.mark.gpu
TOL = 5e-3


def _q():
    import bit_nf4_quantized_pack_b200 as q
    return q


def _codes(packed: np.ndarray, numel: int) -> np.ndarray:
    hi, lo = packed >> 4, packed & 15
    return np.stack([hi, lo], axis=1).ravel()[:numel]


@pytest.mark.parametrize("numel,dtype", [(64 * 37, torch.bfloat16), (64 * 37 + 5, torch.bfloat16),
                                         (64 * 512 + 33, torch.float32), (1, torch.float32)])
def test_int4_quantize_bit_exact(numel, dtype):
    q = _q()
    rng = np.random.default_rng(numel)
    w = rng.normal(0, 0.02, numel).astype(np.float32)
    if numel > 200:
        w[64:128] = 0.0                        # an all-zero block
        w[128:192] = np.arange(64) % 15 - 7.0  # amax 7 -> s = 1: exact ties below
        w[128:136] = [0.5, 1.5, -2.5, 3.5, -0.5, 6.5, -6.5, 2.5]
    if dtype == torch.bfloat16:
        w = S.f32_to_bf16_values(w)
    wq = q.quantize(to_dev(w, dtype), codebook="int4")
    codes, scales = int4_quantize(w)
    assert np.array_equal(wq.absmax.cpu().numpy().view(np.uint32), scales.view(np.uint32))
    packed = wq.packed.cpu().numpy()
    assert np.array_equal(_codes(packed, numel), codes)
    if numel % 2:
        assert packed[-1] & 15 == 8            # odd tail padded with code 8
    dq = q.dequantize(wq)
    assert np.array_equal(to_np(dq), int4_dequantize(codes, scales))


def test_int4_rejects_double_quant():
    q = _q()
    with pytest.raises(ValueError):
        q.NF4Weight.empty((64, 64), True, "cuda", codebook=1)


def _int4_case(seed, M, K, N, r):
    lin = S.random_case(seed, M, K, N, r)
    codes, scales = int4_quantize(lin.W.ravel())
    w_hat = int4_dequantize(codes, scales).reshape(K, N)
    return lin, w_hat


@pytest.mark.parametrize("M,K,N,r", [(200, 320, 384, 16), (129, 256, 512, 8), (4, 640, 576, 16)])
def test_int4_linear_parity(M, K, N, r):
    q = _q()
    lin, w_hat = _int4_case(300 + M, M, K, N, r)
    lin.dY = S.normal(301 + M, M, 4, (M, N), 1.0)
    c = 32.0 / r
    wq = q.quantize(to_dev(lin.W), codebook="int4")
    Xt, At, Bt = to_dev(lin.X), to_dev(lin.A), to_dev(lin.B)
    Y, Zc = q.linear_forward(Xt, wq, At, Bt, c)
    Yr, _ = lora_forward(lin.X, w_hat, lin.A, lin.B, c)
    assert rel_fro(to_np(Y), Yr) <= TOL
    if M > 16:
        dX, dA, dB = q.linear_backward(to_dev(lin.dY), Xt, Zc, wq, At, Bt, c)
        dXr, dAr, dBr = lora_backward(lin.dY, lin.X, w_hat, lin.A, lin.B, c)
        for got, ref in ((dX, dXr), (dA, dAr), (dB, dBr)):
            assert rel_fro(to_np(got), ref) <= TOL


def test_int4_merge():
    q = _q()
    lin, w_hat = _int4_case(77, 4, 256, 320, 16)
    wq = q.quantize(to_dev(lin.W), codebook="int4")
    got = to_np(q.merge(wq, to_dev(lin.A), to_dev(lin.B), 2.0))
    ref = merge_bf16(w_hat, lin.A, lin.B, 2.0)
    ex = merge_exact(w_hat, lin.A, lin.B, 2.0)
    _, e = np.frexp(np.maximum(np.abs(ex), 1e-30))
    assert np.all(np.abs(got - ref) <= np.ldexp(1.0, e - 8))

"""GPU parity at the workload configurations' own shapes, element by element.

Configurations 1 and 2 are covered in test_gpu_linear.py.  Here:

* config 3: the decode GEMV (M in {1, 4, 16}) on both the 4096 x 11008 and
  the 11008 x 4096 weight, double quantization, r = 16: the whole quantized
  state bit for bit, then all of Y and Zc against the oracle's fp64 forward on
  the oracle's own full quantization of the same weight.
* config 4: the seven linears of a 7B decoder layer (q, k, v, o 4096 x 4096;
  gate, up 4096 x 11008; down 11008 x 4096) with 0.1% outliers at 10 sigma,
  r = 64, alpha = 16, double quantization, M = 4096 tokens: the whole state,
  and all of Y, dX, dA and dB.
* config 5: the 65B MLP slice (8192 x 22016 and 22016 x 8192) with double
  quantization, M = 4096, r = 64: the whole scale state (every code8, s2 and
  the offset), the packed bytes of the sampled blocks, sampled columns of Y
  and of dX, all of dA and dB, and sampled rows of the merged weight.

Every output is held to three bounds (tests/_gpu_util.py): the whole-matrix
relative Frobenius error of 5e-3, and the worst row's and the worst 128 x 128
tile's relative error, so that a few wrong outputs cannot hide in a large norm.
"""
import numpy as np
import pytest
import torch

from inputs import synthetic as S
from oracle import nf4
from oracle.linear import lora_backward, lora_forward
from tests._gpu_util import OracleWeight, assert_close, assert_state_equal, to_dev, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _q():
    import bit_nf4_quantized_pack_b200 as q
    return q


@pytest.mark.parametrize("which", [0, 1], ids=["4096x11008", "11008x4096"])
def test_config3_gemv_full_output(which):
    q = _q()
    wl = S.config3()
    lin = wl.linears[which]
    ow = OracleWeight(lin.W, True)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    assert_state_equal(wq, ow)
    At, Bt = to_dev(lin.A), to_dev(lin.B)
    for M in (1, 4, 16):
        X = np.ascontiguousarray(lin.X[:M])
        Y, Zc = q.linear_forward(to_dev(X), wq, At, Bt, wl.c)
        Yr, Zr = lora_forward(X, ow.w_hat, lin.A, lin.B, wl.c)
        rep = assert_close(f"Y M={M}", to_np(Y), Yr)
        assert_close(f"Zc M={M}", to_np(Zc), wl.c * Zr)
        print(f"config 3 {lin.K}x{lin.N} M={M}: Y error {rep}")


@pytest.mark.parametrize("i", range(len(S.LAYER7B)), ids=[n for n, _, _ in S.LAYER7B])
def test_config4_decoder_layer_linear(i):
    """One linear of config 4, drawn exactly as inputs.synthetic.config4 draws
    it (same seeds), with everything compared in full."""
    q = _q()
    wl = S.config4(with_data=False)          # r, alpha, c of the configuration
    name, K, N = S.LAYER7B[i]
    lin = S.make_linear(4, i, name, 4096, K, N, 0.02, wl.r, outlier_frac=0.001,
                        outlier_value=0.2)
    # the outliers (+-0.2 before the bf16 rounding, 10 sigma) are all there
    assert 0.0009 * K * N < np.count_nonzero(np.abs(lin.W) > 0.15) < 0.0011 * K * N
    ow = OracleWeight(lin.W, True)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    assert_state_equal(wq, ow)
    Xt, At, Bt = to_dev(lin.X), to_dev(lin.A), to_dev(lin.B)
    Y, Zc = q.linear_forward(Xt, wq, At, Bt, wl.c)
    dX, dA, dB = q.linear_backward(to_dev(lin.dY), Xt, Zc, wq, At, Bt, wl.c)
    Yr, Zr = lora_forward(lin.X, ow.w_hat, lin.A, lin.B, wl.c)
    assert_close("Y", to_np(Y), Yr)
    assert_close("Zc", to_np(Zc), wl.c * Zr)
    del Y, Yr
    dXr, dAr, dBr = lora_backward(lin.dY, lin.X, ow.w_hat, lin.A, lin.B, wl.c)
    assert_close("dX", to_np(dX), dXr)
    assert_close("dA", to_np(dA), dAr)
    assert_close("dB", to_np(dB), dBr)


def test_config5_mlp_slice_with_double_quant():
    """Both 65B MLP weights with double quantization.  The oracle computes the
    full first-level scales and their double quantization (every code8, s2
    and the offset are compared), and decodes only the blocks that the sampled
    outputs need: for a column j of Y, the block of column j in every row k;
    for a column k of dX, every block of row k."""
    q = _q()
    wl = S.config5(with_data=False)
    rng = np.random.default_rng(5)
    for i, (name, K, N) in enumerate([("up", 8192, 22016), ("down", 22016, 8192)]):
        lin = S.make_linear(5, i, name, 4096, K, N, 0.015, wl.r)
        X, W, A, B, G, c = lin.X, lin.W, lin.A, lin.B, lin.dY, wl.c
        bpr = N // 64
        absmax = nf4.block_scales(W)
        code8, s2, off = nf4.double_quantize(absmax)
        a_dec = nf4.decode_scales(absmax.size, code8=code8, s2=s2, offset=off)
        wq = q.quantize(to_dev(W), double_quant=True)
        assert np.array_equal(wq.code8.cpu().numpy(), code8), "scale codes differ"
        assert np.array_equal(wq.s2.cpu().numpy().view(np.uint32), s2.view(np.uint32)), "s2 differs"
        assert wq.offset.cpu().numpy().view(np.uint32)[0] == np.float32(off).view(np.uint32)
        Xt, At, Bt = to_dev(X), to_dev(A), to_dev(B)
        Y, Zc = q.linear_forward(Xt, wq, At, Bt, c)
        dX, dA, dB = q.linear_backward(to_dev(G), Xt, Zc, wq, At, Bt, c)
        X64, G64, A64, B64 = (np.asarray(t, np.float64) for t in (X, G, A, B))
        Z = X64 @ A64
        dZ = c * (G64 @ B64.T)
        packed_gpu = wq.packed

        def decoded(block, blocks):
            """Oracle decode of a sub-matrix whose 64-blocks are `blocks` (in
            order), with the double-quantized decode scales of those blocks;
            its packed bytes are checked against the GPU's as well."""
            codes, am = nf4.quantize_nf4(np.ascontiguousarray(block, np.float32).ravel())
            assert np.array_equal(am, absmax[blocks])
            payload, n = nf4.pack_codes(codes)
            byte_idx = (blocks[:, None] * 32 + np.arange(32)[None, :]).ravel()
            got = packed_gpu[torch.from_numpy(byte_idx).to(packed_gpu.device)].cpu().numpy()
            assert np.array_equal(got, payload), "packed bytes differ"
            return nf4.dequantize(payload, n, a_dec[blocks]).reshape(block.shape)

        cols = np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, 8)]))
        Ys = to_np(Y[:, torch.from_numpy(cols).to(Y.device)])
        for t, j in enumerate(cols):
            b0 = (j // 64) * 64
            blocks = np.arange(K) * bpr + j // 64
            wcol = decoded(W[:, b0:b0 + 64], blocks)[:, j - b0]
            assert_close(f"{name} Y[:, {j}]", Ys[:, t], X64 @ wcol + c * (Z @ B64[:, j]))
        ks = np.unique(np.concatenate([[0, K - 1], rng.integers(0, K, 8)]))
        dXs = to_np(dX[:, torch.from_numpy(ks).to(dX.device)])
        for t, k in enumerate(ks):
            blocks = k * bpr + np.arange(bpr)
            wrow = decoded(W[k:k + 1, :], blocks).ravel()
            assert_close(f"{name} dX[:, {k}]", dXs[:, t], G64 @ wrow + dZ @ A64[k])
        assert_close(f"{name} dA", to_np(dA), X64.T @ dZ)
        assert_close(f"{name} dB", to_np(dB), c * (Z.T @ G64))
        del Y, dX, Zc
        # the merged weight at full size, on sampled rows: within one bf16 ulp
        # of RN_bf16(W_hat + c A B), nearly all exact
        from oracle.merge import merge_bf16, merge_exact
        merged = q.merge(wq, At, Bt, c)
        ms = to_np(merged[torch.from_numpy(ks).to(merged.device)])
        for t, k in enumerate(ks):
            wrow = decoded(W[k:k + 1, :], k * bpr + np.arange(bpr)).reshape(1, N)
            ref = merge_bf16(wrow, A[k:k + 1], B, c)[0]
            ex = merge_exact(wrow, A[k:k + 1], B, c)[0]
            _, e = np.frexp(np.maximum(np.abs(ex), 1e-30))
            diff = np.abs(ms[t] - ref)
            assert np.all(diff <= np.ldexp(1.0, e - 8)), f"{name} merged row {k}"
            assert np.mean(diff != 0) < 0.01, f"{name} merged row {k}"
        del merged, wq
        torch.cuda.empty_cache()

"""Chained layers with the saved-activation policy (recompute Zc instead of
keeping it), on the GPU.

* the two policies give bit-identical gradients (the recomputation uses the
  forward's kernel and split);
* every layer of the chain matches the fp64 oracle on the inputs that layer
  actually received (relative Frobenius <= 5e-3, as the single-layer tests).
"""
import numpy as np
import pytest
import torch

from inputs import synthetic as S
from oracle.linear import lora_backward, lora_forward
from tests._gpu_util import OracleWeight, rel_fro, to_dev, to_np

pytestmark = pytest.mark.gpu
TOL = 5e-3
WIDTHS = [192, 256, 128, 320]   # K_0 -> N_0 = K_1 -> ... (three layers)
M, R = 200, 16


def _layers(dq=True):
    import bit_nf4_quantized_pack_b200 as q
    from bit_nf4_quantized_pack_b200.chain import Layer
    layers, host = [], []
    for i, (K, N) in enumerate(zip(WIDTHS, WIDTHS[1:])):
        lin = S.random_case(500 + i, M, K, N, R)
        w = q.quantize(to_dev(lin.W), double_quant=dq)
        layers.append(Layer(w, to_dev(lin.A), to_dev(lin.B), 32.0 / R))
        host.append(lin)
    return layers, host


def test_recompute_equals_save_bitwise():
    from bit_nf4_quantized_pack_b200.chain import LinearChain
    layers, host = _layers()
    X = to_dev(host[0].X)
    dY = to_dev(S.normal(901, M, 4, (M, WIDTHS[-1]), 1.0))
    outs = {}
    for policy in ("save", "recompute"):
        ch = LinearChain(layers, policy=policy)
        Y = ch.forward(X)
        dX, grads = ch.backward(dY)
        outs[policy] = (Y, dX, grads)
    (Ys, dXs, gs), (Yr, dXr, gr) = outs["save"], outs["recompute"]
    assert torch.equal(Ys, Yr) and torch.equal(dXs, dXr)
    for (a1, b1), (a2, b2) in zip(gs, gr):
        assert torch.equal(a1, a2) and torch.equal(b1, b2)


def test_chain_layers_match_oracle():
    import bit_nf4_quantized_pack_b200 as q
    from bit_nf4_quantized_pack_b200.chain import LinearChain
    layers, host = _layers(dq=False)
    X = to_dev(host[0].X)
    dY = to_dev(S.normal(902, M, 4, (M, WIDTHS[-1]), 1.0))
    ch = LinearChain(layers, policy="recompute")
    Y = ch.forward(X)
    dX, grads = ch.backward(dY)
    # walk the chain again on the device's own intermediates
    g = dY
    for i in reversed(range(len(layers))):
        L, lin = layers[i], host[i]
        xin = to_np(ch._inputs[i])
        w_hat = OracleWeight(lin.W, False).w_hat
        if i == len(layers) - 1:
            Yr, _ = lora_forward(xin, w_hat, lin.A, lin.B, L.c)
            assert rel_fro(to_np(Y), Yr) <= TOL
        dXr, dAr, dBr = lora_backward(to_np(g), xin, w_hat, lin.A, lin.B, L.c)
        gd, ga, gb = q.linear_backward(g, ch._inputs[i], None, L.w, L.A, L.B, L.c)
        assert torch.equal(ga, grads[i][0]) and torch.equal(gb, grads[i][1])
        for got, ref in ((gd, dXr), (ga, dAr), (gb, dBr)):
            assert rel_fro(to_np(got), ref) <= TOL
        g = gd
    assert torch.equal(g, dX)

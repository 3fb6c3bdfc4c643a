"""Canaries: every output of the library is written through a view into a
larger buffer whose guard regions, before and after the view, hold a
sentinel.  After each call on ragged shapes (odd element counts, partial row
and column tiles, the GEMV and the fused paths, the rank-r recompute) the
guards must be unchanged: no kernel stores outside the rows, columns and
bytes it owns.  Every view starts a multiple of 16 bytes into its buffer, as
the boundary requires."""
import numpy as np
import pytest
import torch

from inputs import synthetic as S
from tests._gpu_util import to_dev

pytestmark = pytest.mark.gpu
PAD = 4096   # guard elements on each side


def _q():
    import bit_nf4_quantized_pack_b200 as q
    return q


class Guarded:
    """n elements at offset PAD of a buffer of n + 2*PAD filled with `fill`."""

    def __init__(self, n, dtype, fill):
        self.n = n
        self.big = torch.full((n + 2 * PAD,), fill, dtype=dtype, device="cuda")
        self.ref = self.big.clone()
        self.t = self.big[PAD:PAD + n]

    def intact(self):
        torch.cuda.synchronize()
        return (torch.equal(self.big[:PAD], self.ref[:PAD])
                and torch.equal(self.big[PAD + self.n:], self.ref[PAD + self.n:]))


@pytest.mark.parametrize("dq", [True, False])
def test_quantize_and_dequantize_stay_inside(dq):
    q = _q()
    numel = 64 * 300 + 5                       # odd: a padded last byte, a ragged block
    rng = np.random.default_rng(31)
    w = S.f32_to_bf16_values(rng.normal(0, 0.02, numel).astype(np.float32))
    W = to_dev(w)
    n1, n2 = q.n1_of(numel), q.n2_of(numel)
    packed = Guarded((numel + 1) // 2, torch.uint8, 0xA5)
    guards = [packed]
    if dq:
        code8 = Guarded(n1, torch.uint8, 0x5A)
        s2 = Guarded(n2, torch.float32, -7.25)
        off = Guarded(1, torch.float32, -7.25)
        wq = q.NF4Weight((numel,), True, packed.t, code8=code8.t, s2=s2.t, offset=off.t)
        guards += [code8, s2, off]
    else:
        absmax = Guarded(n1, torch.float32, -7.25)
        wq = q.NF4Weight((numel,), False, packed.t, absmax=absmax.t)
        guards += [absmax]
    q.quantize(W, double_quant=dq, out=wq)
    out = Guarded(numel, torch.bfloat16, 1234.5)
    q.dequantize(wq, out=out.t)
    guards.append(out)
    assert all(g.intact() for g in guards)
    assert (int(packed.t[-1].item()) & 15) == 7          # the odd tail's pad code


@pytest.mark.parametrize("M,K,N,r", [(200, 320, 384, 16), (129, 256, 192, 8), (300, 512, 192, 64),
                                     (3, 576, 320, 8), (16, 1088, 1344, 64)])
def test_linear_outputs_stay_inside(M, K, N, r):
    q = _q()
    lin = S.random_case(900 + M + K, M, K, N, r)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    Xt, At, Bt = to_dev(lin.X), to_dev(lin.A), to_dev(lin.B)
    Y = Guarded(M * N, torch.bfloat16, 1234.5)
    Zc = Guarded(M * r, torch.bfloat16, 1234.5)
    q.linear_forward(Xt, wq, At, Bt, 2.0, Y=Y.t.view(M, N), Zc=Zc.t.view(M, r))
    assert Y.intact() and Zc.intact()
    if M <= 16:
        return
    G = to_dev(S.normal(902 + M, M, 4, (M, N), 1.0))
    for zc in (Zc.t.view(M, r), None):         # saved Zc, then the recompute policy
        dX = Guarded(M * K, torch.bfloat16, 1234.5)
        dA = Guarded(K * r, torch.float32, -7.25)
        dB = Guarded(r * N, torch.float32, -7.25)
        q.linear_backward(G, Xt, zc, wq, At, Bt, 2.0, dX=dX.t.view(M, K), dA=dA.t.view(K, r),
                          dB=dB.t.view(r, N))
        assert dX.intact() and dA.intact() and dB.intact()


def test_merge_output_stays_inside():
    q = _q()
    K, N, r = 320, 384, 16
    lin = S.random_case(950, 4, K, N, r)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    out = Guarded(K * N, torch.bfloat16, 1234.5)
    q.merge(wq, to_dev(lin.A), to_dev(lin.B), 2.0, out=out.t.view(K, N))
    assert out.intact()

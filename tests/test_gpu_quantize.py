"""GPU parity of qlora_nf4_quantize / qlora_nf4_dequantize against the oracle.

Bit-exact: packed bytes, first-level scales, scale codes, second-level scales,
offset, and the dequantized bf16 weights.
"""
import numpy as np
import pytest
import torch

from inputs import synthetic as S
from oracle import nf4
from tests._gpu_util import OracleWeight, assert_state_equal, bf16_bits, dev, to_dev

pytestmark = pytest.mark.gpu


def _q():
    import bit_nf4_quantized_pack_b200 as q
    return q


def _weights(rng, P, bf16):
    w = (rng.standard_normal(P) * 0.02).astype(np.float32)
    w[rng.random(P) < 0.002] = 0.3
    if P > 256:
        w[128:192] = 0.0                            # an all-zero block
    return S.f32_to_bf16_values(w) if bf16 else w


@pytest.mark.parametrize("P", [1, 2, 7, 63, 64, 65, 127, 1000, 4097, 64 * 256 + 5, 300001])
@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("dq", [False, True])
def test_quantize_dequantize_bit_exact_ragged(P, bf16, dq):
    q = _q()
    rng = np.random.default_rng(P * 7 + bf16 * 3 + dq)
    w = _weights(rng, P, bf16)
    wt = to_dev(w, torch.bfloat16 if bf16 else torch.float32)
    g = q.quantize(wt, double_quant=dq)
    ow = OracleWeight(w, dq)
    assert_state_equal(g, ow)
    out = q.dequantize(g)
    want = nf4.bf16_bits(ow.w_hat.ravel())
    assert np.array_equal(bf16_bits(out).ravel(), want)


def test_config1_tiny_fp32():
    q = _q()
    wl = S.config1()
    W = wl.linears[0].W
    g = q.quantize(to_dev(W, torch.float32), double_quant=False)
    ow = OracleWeight(W, False)
    assert_state_equal(g, ow)
    assert float(g.absmax[5]) == 1.0 and np.all(ow.codes[320:384] == 7)
    assert np.array_equal(bf16_bits(q.dequantize(g)).ravel(), nf4.bf16_bits(ow.w_hat.ravel()))


def _adversarial(a):
    from fractions import Fraction
    vals = [np.float32(a), np.float32(-a)]
    for j in range(15):
        m = (Fraction(nf4.NF4[j]) + Fraction(nf4.NF4[j + 1])) / 2
        t = np.float32(float(Fraction(float(a)) * m))
        for k in range(-3, 4):
            v = t
            for _ in range(abs(k)):
                v = np.nextafter(v, np.float32(np.inf if k > 0 else -np.inf))
            if abs(v) <= a:
                vals.append(v)
    vals = vals[:64]
    vals += [np.float32(0)] * (64 - len(vals))
    return np.array(vals, np.float32)


def test_near_midpoint_blocks_bit_exact():
    q = _q()
    rng = np.random.default_rng(3)
    scales = [1.0, 0.5, 2.0 ** -30, 0.0123456, 1e4] + list(rng.uniform(1e-3, 1, 60))
    w = np.concatenate([_adversarial(np.float32(a)) for a in scales])
    for bf16 in (False, True):
        x = S.f32_to_bf16_values(w) if bf16 else w
        g = q.quantize(to_dev(x, torch.bfloat16 if bf16 else torch.float32), double_quant=False)
        ow = OracleWeight(x, False)
        assert_state_equal(g, ow)


def test_nonfinite_raises_status():
    q = _q()
    for bad in (np.nan, np.inf, -np.inf):
        w = np.zeros(1000, np.float32)
        w[517] = bad
        status = q.new_status()
        q.quantize(to_dev(w, torch.float32), double_quant=True, status=status)
        code, mask = q.status_sync(status)
        assert code == 3 and mask & (1 << 3)
    with pytest.raises(q.QLoRAError):
        w = np.ones(100, np.float32)
        w[3] = np.nan
        q.quantize(to_dev(w, torch.float32), double_quant=False)


def test_bad_padding_raises_status():
    q = _q()
    w = np.linspace(-1, 1, 101).astype(np.float32)
    g = q.quantize(to_dev(w, torch.float32), double_quant=False)
    last = int(g.packed[-1])
    assert last & 15 == 7
    g.packed[-1] = (last & 0xF0) | 3
    status = q.new_status()
    q.dequantize(g, status=status)
    code, _ = q.status_sync(status)
    assert code == 4


def test_full_size_projection_double_quant():
    q = _q()
    W = S.config2(M=1).linears[0].W
    g = q.quantize(to_dev(W), double_quant=True)
    ow = OracleWeight(W, True)
    assert_state_equal(g, ow)
    out = q.dequantize(g)
    assert np.array_equal(bf16_bits(out).ravel(), nf4.bf16_bits(ow.w_hat.ravel()))


@pytest.mark.slow
def test_full_size_65b_mlp_sampled():
    """8192 x 22016: every block scale and the exact offset, plus sampled blocks."""
    q = _q()
    W = S.make_linear(5, 0, "up", 1, 8192, 22016, 0.015, 64, with_x=False, with_dy=False).W
    wt = to_dev(W)
    g = q.quantize(wt, double_quant=True)
    del wt
    flat = W.ravel()
    n1 = flat.size // 64
    # every block scale through the oracle, in chunks
    scales = nf4.block_scales(flat)
    code8, s2, off = nf4.double_quantize(scales)
    assert g.offset.cpu().numpy().view(np.uint32)[0] == np.float32(off).view(np.uint32)
    assert np.array_equal(g.s2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    assert np.array_equal(g.code8.cpu().numpy(), code8)
    rng = np.random.default_rng(0)
    blocks = np.unique(np.concatenate([[0, n1 - 1], rng.integers(0, n1, 4000)]))
    packed = g.packed.cpu().numpy()
    for b in blocks:
        codes, _ = nf4.quantize_nf4(flat[b * 64:(b + 1) * 64])
        payload, _ = nf4.pack_codes(codes)
        assert np.array_equal(packed[b * 32:(b + 1) * 32], payload), b


@pytest.mark.parametrize("nblk", [128 * 3, 128 * 5 + 37])
def test_double_quant_bf16_scales_spread_over_binades(nblk):
    """bf16 weights whose block scales spread from bf16 subnormals to near the
    largest bf16, mixed inside every group of 16 consecutive blocks: the
    encoder's exponent bins then meet, within one warp, scales close to the
    warp's largest and scales far below it.  Whole state, DQ offset
    included, bit-exact against the oracle (whole 8192-element chunks plus a
    ragged tail of blocks)."""
    q = _q()
    rng = np.random.default_rng(nblk)
    e = rng.integers(-133, 127, nblk).astype(np.float64)
    m = rng.integers(128, 256, nblk) / 128.0
    sc = S.f32_to_bf16_values((m * 2.0 ** e).astype(np.float32))
    sc[rng.random(nblk) < 0.5] = np.float32(0.0078125)   # a cluster of equal scales
    w = np.zeros(64 * nblk, np.float32)
    w[::64] = sc
    w[1::64] = S.f32_to_bf16_values(-sc * np.float32(0.5))
    w[2::64] = S.f32_to_bf16_values(sc * np.float32(0.3))
    g = q.quantize(to_dev(w, torch.bfloat16), double_quant=True)
    ow = OracleWeight(w, True)
    assert_state_equal(g, ow)
    assert np.array_equal(nf4.block_scales(w), sc)


@pytest.mark.parametrize("scales", [
    [1.0, 1.0 + 2.0 ** -23],                        # exact tie -> even (1.0)
    [1.0 + 2.0 ** -23, 1.0 + 2.0 ** -22],           # exact tie -> even (upper)
    [2.0 ** -149, 2.0 ** -149, 2.0 ** -148],        # subnormal scales
    [1e-30, 1.0, 3.0],                              # > 64 binades apart: wide path
    [1e-38, 3e38],                                  # extreme spread
    [0.037] * 1000,                                 # equal scales
    [2.0 ** 24] + [1.0] * 4095,                     # naive fp32 running sum would lose these
])
def test_double_quant_offset_is_the_exact_mean(scales):
    """Blocks whose absmax equals each listed scale; the DQ offset must equal
    the oracle's exactly rounded mean bit for bit."""
    q = _q()
    sc = np.array(scales, np.float32)
    w = np.zeros(64 * sc.size, np.float32)
    w[::64] = sc                                    # one element per block carries the scale
    w[1::64] = -sc * np.float32(0.5)
    g = q.quantize(to_dev(w, torch.float32), double_quant=True)
    ow = OracleWeight(w, True)
    assert_state_equal(g, ow)
    assert np.array_equal(nf4.block_scales(w), sc)

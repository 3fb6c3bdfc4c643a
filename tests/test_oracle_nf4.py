"""Pins of the NF4 oracle against what the pages and plain mathematics fix.

Sources: "QLoRA：冻结的 4-bit 权重怎样参与一次微调", §NF4 保存的是索引而不是均匀
整数值, §从 NF4 索引打包成字节, §Double Quantization 压缩的是 Scale,
§Merge 后还是不是训练时的函数.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4


def test_table_is_fp32_exact_sorted_with_exact_zero():
    t = np.array(nf4.NF4)
    assert t.size == 16
    assert np.all(np.diff(t) > 0)
    assert np.all(t.astype(np.float32).astype(np.float64) == t)
    # 7 negatives, one exact zero at index 7, 8 positives (printed table)
    assert np.sum(t < 0) == 7 and t[7] == 0.0 and np.sum(t > 0) == 8
    assert t[0] == -1.0 and t[15] == 1.0


def test_worked_example(golden):
    g = golden("nf4_worked_example.json")
    codes, restored, scale = nf4.encode_block(g["block"])
    assert codes == g["codes"] and scale == g["scale"]
    assert restored == g["restored"]
    for r, p in zip(restored, g["restored_printed_approx"]):
        assert abs(r - p) < 5e-9
    payload, length = nf4.pack_codes(codes)
    assert bytes(payload).hex() == g["payload_hex"] and length == 4
    assert list(nf4.unpack_codes(payload, length)) == g["codes"]
    # vectorised path agrees
    c2, s2 = nf4.quantize_nf4(np.array(g["block"], dtype=np.float32))
    assert list(c2) == g["codes"] and float(s2[0]) == g["scale"]


def test_odd_roundtrip_and_all_zero(golden):
    g = golden("nf4_worked_example.json")
    odd = g["odd_roundtrip_codes"]
    payload, length = nf4.pack_codes(odd)
    assert payload.size == 2 and (int(payload[-1]) & 15) == 7
    assert list(nf4.unpack_codes(payload, length)) == odd
    codes, _, scale = nf4.encode_block(g["all_zero_block"])
    assert codes == g["all_zero_codes"] and scale == g["all_zero_scale"]
    c2, s2 = nf4.quantize_nf4(np.zeros(64, np.float32))
    assert np.all(c2 == 7) and s2[0] == 1.0


def test_merge_requantization(golden):
    g = golden("merge_requant_example.json")
    w_hat, A, B, c, x = g["w_hat"], g["A"], g["B"], g["c"], g["x"]
    cab = [c * a * B for a in A]
    assert all(abs(u - v) < 1e-15 for u, v in zip(cab, g["cAB"]))
    merged = [w + d for w, d in zip(w_hat, cab)]
    assert all(abs(u - v) < 1e-15 for u, v in zip(merged, g["merged"]))
    assert abs(sum(xi * wi for xi, wi in zip(x, merged)) - g["merged_output"]) < 1e-12
    codes, restored, scale = nf4.encode_block(g["merged"])
    assert codes == g["requant_codes"] and scale == g["requant_scale"]
    tol = g["approx_abs_tol"]
    assert abs(restored[1] - g["requant_second_weight_approx"]) < tol
    assert abs(sum(xi * wi for xi, wi in zip(x, restored)) - g["requant_output_approx"]) < tol
    assert not math.isclose(restored[1], g["merged"][1])


def _brute_exact(block):
    """Exact-rational nearest code, ties to the smaller index (slow)."""
    a = max(abs(Fraction(float(v))) for v in block)
    s = a if a else Fraction(1)
    out = []
    for v in block:
        n = Fraction(float(v)) / s
        best, bd = None, None
        for j, cj in enumerate(nf4.NF4):
            d = abs(n - Fraction(cj))
            if bd is None or d < bd:
                best, bd = j, d
        out.append(best)
    return out


def test_vectorised_matches_page_rule_random_ragged():
    rng = np.random.default_rng(1)
    for P in (1, 2, 3, 63, 64, 65, 127, 130, 257):
        w = (rng.standard_normal(P) * 0.02).astype(np.float32)
        w[rng.random(P) < 0.05] = 0.0
        codes, absmax = nf4.quantize_nf4(w)
        for b in range(absmax.size):
            blk = w[b * 64:(b + 1) * 64]
            c_ref, _, s_ref = nf4.encode_block(blk)
            assert list(codes[b * 64:b * 64 + blk.size]) == c_ref
            assert float(absmax[b]) == s_ref


def _adversarial_block(rng, a):
    """fp32 neighbours (+-2 ulp) of a*m_j for every NF4 midpoint m_j."""
    mids = [(Fraction(nf4.NF4[j]) + Fraction(nf4.NF4[j + 1])) / 2 for j in range(15)]
    vals = [np.float32(a)]
    for m in mids:
        t = np.float32(float(Fraction(float(a)) * m))
        for k in range(-2, 3):
            v = t
            step = np.inf if k > 0 else -np.inf
            for _ in range(abs(k)):
                v = np.nextafter(v, np.float32(step))
            if abs(v) <= a:
                vals.append(v)
    return np.array(vals[:64], dtype=np.float32)


def test_exact_rational_bruteforce_including_near_midpoints():
    rng = np.random.default_rng(2)
    scales = [1.0, 0.5, 0.3, 2.0 ** -20, 0.0123456, 3.0e4]
    scales += list(np.abs(rng.standard_normal(10)).astype(np.float32) * 0.05 + 1e-3)
    for a in scales:
        a = np.float32(a)
        blk = _adversarial_block(rng, a)
        codes, absmax = nf4.quantize_nf4(blk)
        assert list(codes) == _brute_exact(blk)
        assert absmax[0] == np.max(np.abs(blk))
    for _ in range(20):
        blk = (rng.standard_normal(64) * rng.uniform(1e-3, 1.0)).astype(np.float32)
        codes, _ = nf4.quantize_nf4(blk)
        assert list(codes) == _brute_exact(blk)


def test_exact_ties_go_to_the_smaller_index():
    # with a = 1, w equal to an fp32-representable midpoint is an exact tie
    for j in range(15):
        m = (nf4.NF4[j] + nf4.NF4[j + 1]) / 2
        if float(np.float32(m)) != m:
            continue
        codes, _, _ = nf4.encode_block([1.0, m])
        assert codes[1] == j, (j, m)
        c2, _ = nf4.quantize_nf4(np.array([1.0, m], np.float32))
        assert c2[1] == j


@pytest.mark.parametrize("length", list(range(0, 131)))
def test_pack_unpack_roundtrip(length):
    rng = np.random.default_rng(length)
    codes = rng.integers(0, 16, size=length)
    payload, n = nf4.pack_codes(codes)
    assert n == length and payload.size == (length + 1) // 2
    # high nibble first
    for i in range(length):
        byte = int(payload[i // 2])
        assert (byte >> 4 if i % 2 == 0 else byte & 15) == codes[i]
    assert np.array_equal(nf4.unpack_codes(payload, n), codes.astype(np.uint8))


def test_unpack_rejects_bad_length_and_padding():
    payload, n = nf4.pack_codes([1, 2, 3])
    with pytest.raises(nf4.PaddingError):
        nf4.unpack_codes(payload, 5)
    with pytest.raises(nf4.PaddingError):
        nf4.unpack_codes(payload[:1], 3)
    bad = payload.copy()
    bad[-1] = (bad[-1] & 0xF0) | 3
    with pytest.raises(nf4.PaddingError):
        nf4.unpack_codes(bad, 3)
    with pytest.raises(ValueError):
        nf4.pack_codes([16])


def test_nonfinite_and_empty_rejected():
    with pytest.raises(nf4.NonFiniteError):
        nf4.encode_block([1.0, float("nan")])
    with pytest.raises(nf4.NonFiniteError):
        nf4.encode_block([])
    with pytest.raises(nf4.NonFiniteError):
        nf4.quantize_nf4(np.array([0.0, np.inf], np.float32))
    with pytest.raises(ValueError):
        nf4.quantize_nf4(np.array([], np.float32))


def test_bit_budget(golden):
    g = golden("bit_budget.json")
    for P in (64 * 256 * 4096, 64 * 256 * 65536):
        no = nf4.bit_budget(P, False) / P
        dq = nf4.bit_budget(P, True) / P
        assert no == g["bits_no_dq_asymptote"]
        assert abs(dq - g["bits_dq_asymptote"]) == 32 / P       # the global offset
    big = 64 * 256 * (1 << 24)
    assert abs(nf4.bit_budget(big, True) / big - g["bits_dq_asymptote"]) < 1e-9
    assert g["bits_no_dq_asymptote"] - g["bits_dq_asymptote"] == g["saving_per_weight"]
    assert abs((8 / 64 + 32 / (64 * 256)) - g["scale_bits_dq_paper_approx"]) < 5e-4
    # the buffers the oracle produces have exactly the counted sizes
    w = np.random.default_rng(0).standard_normal(1000).astype(np.float32)
    codes, absmax = nf4.quantize_nf4(w)
    payload, _ = nf4.pack_codes(codes)
    code8, s2, off = nf4.double_quantize(absmax)
    bits = 8 * payload.size + 8 * code8.size + 32 * s2.size + 32
    assert bits == nf4.bit_budget(1000, True)
    assert 8 * payload.size + 32 * absmax.size == nf4.bit_budget(1000, False)


def _bf16_neighbours(x):
    """The two bf16 values around x (exact, by enumeration of the bf16 grid)."""
    f = np.float32(x)
    u = int(np.array(f).view(np.uint32)) & 0xFFFF0000
    lo = np.array(np.uint32(u)).view(np.float32).item()
    hi = np.array(np.uint32(u + 0x10000)).view(np.float32).item()
    return lo, hi


def test_round_to_bf16_ties_and_random():
    one = 1.0
    assert nf4.round_to_bf16(one + 2 ** -8) == 1.0                 # tie -> even
    assert nf4.round_to_bf16(one + 3 * 2 ** -8) == one + 2 ** -6     # tie -> even
    assert nf4.round_to_bf16(one + 2 ** -8 + 2 ** -40) == one + 2 ** -7   # not a tie
    assert nf4.round_to_bf16(-(one + 2 ** -8 + 2 ** -40)) == -(one + 2 ** -7)
    rng = np.random.default_rng(3)
    xs = rng.standard_normal(2000) * 10.0 ** rng.uniform(-30, 30, 2000)
    out = nf4.round_to_bf16(xs)
    for x, r in zip(xs, out):
        lo, hi = sorted(_bf16_neighbours(abs(x)))
        if not lo <= abs(x) <= hi:
            lo, hi = sorted(_bf16_neighbours(np.nextafter(np.float32(abs(x)), np.float32(0))))
        dl, dh = abs(Fraction(abs(x)) - Fraction(lo)), abs(Fraction(hi) - Fraction(abs(x)))
        want = lo if dl < dh else hi if dh < dl else None
        if want is not None:
            assert abs(r) == want, (x, r, lo, hi)


def test_dequantize_worked_examples(golden):
    g = golden("backward_worked_example.json")
    w = nf4.dequantize(np.frombuffer(bytes.fromhex(g["packed_hex"]), np.uint8), 2,
                       np.array([g["scale"]], np.float32))
    assert list(w) == g["w_hat"]
    e = golden("nf4_worked_example.json")
    codes, absmax = nf4.quantize_nf4(np.array(e["block"], np.float32))
    payload, n = nf4.pack_codes(codes)
    w = nf4.dequantize(payload, n, absmax)
    for got, r in zip(w, e["restored"]):
        lo, hi = sorted(_bf16_neighbours(abs(r))) if r else (0.0, 0.0)
        assert abs(got) in (lo, hi) and abs(abs(got) - abs(r)) <= abs(r) * 2 ** -8


def test_block_scales_is_the_scale_step_of_quantize():
    rng = np.random.default_rng(13)
    for P in (1, 64, 65, 1000):
        w = (rng.standard_normal(P) * 0.02).astype(np.float32)
        if P > 64:
            w[:64] = 0
        _, s = nf4.quantize_nf4(w)
        assert np.array_equal(nf4.block_scales(w), s)
    with pytest.raises(nf4.NonFiniteError):
        nf4.block_scales(np.array([1.0, np.nan], np.float32))


def test_round_to_bf16_subnormal_and_overflow():
    """Round to nearest even at the ends of the bf16 range: subnormals are
    multiples of 2^-133 (fp32-exact inputs checked against the enumerated
    bf16 grid), and past the largest bf16 value (2 - 2^-7) * 2^127 a tie
    rounds to even, which is the overflow to infinity."""
    rng = np.random.default_rng(21)
    k = rng.integers(1, 1 << 23, 3000)
    xs = np.ldexp(k.astype(np.float64), -149)          # fp32 subnormals: exact
    xs = np.concatenate([xs, np.ldexp(rng.uniform(1, 2, 500), rng.integers(-130, -120, 500))])
    xs = xs.astype(np.float32).astype(np.float64)      # keep them fp32-exact
    out = nf4.round_to_bf16(xs)
    for x, r in zip(xs, out):
        lo, hi = _bf16_neighbours(x)
        dl, dh = Fraction(x) - Fraction(lo), Fraction(hi) - Fraction(x)
        if dl < dh:
            assert r == lo, x
        elif dh < dl:
            assert r == hi, x
        else:   # tie: the even bf16 pattern
            even = lo if (int(np.array(np.float32(lo)).view(np.uint32)) >> 16) % 2 == 0 else hi
            assert r == even, x
    top = (2.0 - 2.0 ** -7) * 2.0 ** 127                # largest bf16, odd mantissa
    ulp = 2.0 ** 120
    assert nf4.round_to_bf16(top + ulp / 4) == top
    assert nf4.round_to_bf16(top + ulp / 2) == np.inf   # tie -> even -> 2^128 overflows
    assert nf4.round_to_bf16(-(top + 0.75 * ulp)) == -np.inf
    assert nf4.round_to_bf16(2.0 ** -134) == 0.0        # half the smallest subnormal: tie -> 0
    assert nf4.round_to_bf16(3 * 2.0 ** -134) == 2 * 2.0 ** -133   # tie -> even


def test_ragged_tail_block_is_its_own_block():
    """The last block holds only the tail (the page's blocks of 64 of the
    flattening, the last one shorter): a large element just before it does
    not enter its scale, and an all-zero tail gets scale 1 and code 7."""
    w = np.full(64 + 5, 0.01, np.float32)
    w[63] = 10.0
    w[64:] = [0.2, -0.4, 0.0, 0.1, 0.05]
    codes, absmax = nf4.quantize_nf4(w)
    assert absmax[1] == np.float32(0.4) and nf4.block_scales(w)[1] == np.float32(0.4)
    tail_codes, _, tail_scale = nf4.encode_block(w[64:])
    assert list(codes[64:]) == tail_codes and tail_scale == np.float32(0.4)
    w[64:] = 0.0
    codes, absmax = nf4.quantize_nf4(w)
    assert absmax[1] == 1.0 and nf4.block_scales(w)[1] == 1.0
    assert np.all(codes[64:] == 7)


def test_encode_block_exact_near_midpoints():
    """The per-block rule in Python doubles agrees with exact rational
    arithmetic on fp32 neighbours of every NF4 midpoint."""
    rng = np.random.default_rng(22)
    for a in (1.0, 0.3, 2.0 ** -20, 0.0123456, 3.0e4):
        blk = _adversarial_block(rng, np.float32(a))
        codes, _, _ = nf4.encode_block(blk)
        assert codes == _brute_exact(blk)


def test_dequantize_rejects_nonfinite_scale():
    """A non-finite reconstruction is an error (the page's decode check)."""
    payload, n = nf4.pack_codes(np.array([7, 9, 3, 15], dtype=np.uint8))
    with pytest.raises(nf4.NonFiniteError):
        nf4.dequantize(payload, n, np.array([np.inf], dtype=np.float32))
    with pytest.raises(nf4.NonFiniteError):
        nf4.dequantize(payload, n, np.array([np.nan], dtype=np.float32))

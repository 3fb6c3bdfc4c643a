"""Pins of the double-quantization oracle.

Sources: "QLoRA：冻结的 4-bit 权重怎样参与一次微调" §Double Quantization 压缩的是
Scale (mean offset, block 256, fp32 second-level scale, signed 8-bit dynamic
codebook, error C_j * delta_a with codes unchanged); "精读笔记 · QLoRA" §3.2.
The 8-bit codebook's values are this build's own definition (the pages print
none): its structure is pinned here, its values are not ("parity unpinned").
"""
from fractions import Fraction

import numpy as np

from oracle import nf4


def test_codebook_structure():
    t = nf4.dq_codebook()
    assert t.dtype == np.float32 and t.size == 256
    assert t[0x00] == 0.0 and t[0x80] == 0.0
    assert len(set(t.tolist())) == 255
    assert t[0x7F] == 1.0 and t[0xFF] == -1.0
    pos = t[1:128]
    assert np.all(np.diff(pos) > 0)                       # monotone within a sign
    assert np.all(t[0x81:0x100] == -pos)                  # sign bit mirrors
    assert np.all(np.abs(t) <= 1.0)
    # decades: indices 64..127 cover (0.1, 1], 32..63 cover (0.01, 0.1], ...
    assert np.all((pos[63:] > np.float32(0.1)) & (pos[63:] <= 1))
    assert np.all((pos[31:63] > np.float32(0.01)) & (pos[31:63] <= np.float32(0.1)))
    assert t[63] == np.float32(0.1) and t[1] == np.float32(1e-6)
    # not FP8 E4M3: E4M3's largest finite value is 448, its grid is binary
    assert np.float32(0.1) in t and np.max(np.abs(t)) != 448.0


def _mean_by_fraction(v):
    s = sum(Fraction(float(x)) for x in v) / len(v)
    # nearest fp32 by bracketing (independent of the oracle's rounding helper)
    f = np.float32(float(s))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    d = [abs(Fraction(float(c)) - s) for c in cands]
    best = min(d)
    winners = [c for c, dd in zip(cands, d) if dd == best]
    if len(winners) == 1:
        return winners[0]
    even = [c for c in winners if (int(np.array(c).view(np.uint32)) & 1) == 0]
    return even[0]


def test_exact_mean_closed_forms_and_ties():
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -23)
    assert nf4.exact_mean_f32([one, one + ulp]) == one               # tie -> even
    assert nf4.exact_mean_f32([one + ulp, one + 2 * ulp]) == one + 2 * ulp
    assert nf4.exact_mean_f32(np.full(1000, 0.037, np.float32)) == np.float32(0.037)
    assert nf4.exact_mean_f32([1.0, 2.0, 4.0]) == np.float32(7.0 / 3.0)
    # a naive fp32 running sum loses the small terms; the exact mean does not
    v = np.array([2.0 ** 24] + [1.0] * 4095, np.float32)
    naive = np.float32(0)
    for x in v:
        naive = np.float32(naive + x)
    exact = np.float32((2.0 ** 24 + 4095) / 4096)
    assert nf4.exact_mean_f32(v) == exact and np.float32(naive / 4096) != exact
    # subnormals and the largest finite value
    tiny = np.float32(2.0 ** -149)
    assert nf4.exact_mean_f32([tiny, tiny, tiny]) == tiny
    big = np.finfo(np.float32).max
    assert nf4.exact_mean_f32([big, big]) == big


def test_exact_mean_random_against_fractions():
    rng = np.random.default_rng(5)
    for n in (1, 2, 3, 17, 300, 1001):
        v = np.abs(rng.standard_normal(n) * 10.0 ** rng.uniform(-8, 3, n)).astype(np.float32)
        assert nf4.exact_mean_f32(v) == _mean_by_fraction(v)


def _brute_code8(c, s2):
    table = nf4.dq_codebook()
    x = Fraction(float(c)) / Fraction(float(s2))
    best_u, bd, bv = None, None, None
    for u in range(256):
        v = Fraction(float(table[u]))
        d = abs(x - v)
        # ties -> the smaller value; equal values (the two zeros) -> code 0x00
        if bd is None or d < bd or (d == bd and (v < bv or (v == bv and u < best_u))):
            best_u, bd, bv = u, d, v
    return best_u


def test_double_quantize_bruteforce_ragged():
    rng = np.random.default_rng(6)
    for n1 in (1, 5, 256, 257, 700):
        a = np.abs(rng.standard_normal(n1) * 0.02 + 0.05).astype(np.float32)
        a[rng.random(n1) < 0.05] = 1.0                     # all-zero blocks keep scale 1
        code8, s2, off = nf4.double_quantize(a)
        assert s2.size == -(-n1 // 256) and code8.size == n1
        assert off == nf4.exact_mean_f32(a)
        c = (a - off).astype(np.float32)
        for i in range(n1):
            g = i // 256
            grp = c[g * 256:(g + 1) * 256]
            want_s2 = np.max(np.abs(grp)) if np.max(np.abs(grp)) > 0 else np.float32(1)
            assert s2[g] == want_s2
            assert code8[i] == _brute_code8(c[i], s2[g]), i


def test_double_quantize_exact_midpoint_ties():
    table = nf4.dq_codebook()
    vals = sorted(set(table.astype(np.float64).tolist()))
    # scales whose centred values sit exactly on T8 midpoints (s2 = 1 group)
    rng = np.random.default_rng(7)
    picks = rng.choice(len(vals) - 1, size=40, replace=False)
    mids = []
    for k in picks:
        m = (vals[k] + vals[k + 1]) / 2
        if float(np.float32(m)) == m:
            mids.append(np.float32(m))
    assert mids, "need fp32-exact midpoints"
    # build a = c + offset with offset 0: include +1 and -1 so s2 = 1, mean 0
    c = np.array([1.0, -1.0] + mids + [-x for x in mids], np.float32)
    code8, s2, off = nf4.double_quantize(c)
    assert off == 0.0 and s2[0] == 1.0
    for i, x in enumerate(c):
        assert code8[i] == _brute_code8(x, s2[0])
        if x in mids:       # a tie resolves to the smaller value
            lo = max(v for v in vals if v < x)
            assert table[code8[i]] == np.float32(lo)


def test_equal_group_decodes_to_offset_and_error_bound():
    a = np.full(300, 0.0421, np.float32)
    code8, s2, off = nf4.double_quantize(a)
    dec = nf4.decode_scales(300, code8=code8, s2=s2, offset=off)
    assert np.all(code8 == 0) and np.all(s2 == 1.0) and np.all(dec == a)
    rng = np.random.default_rng(8)
    a = np.abs(rng.standard_normal(5000) * 0.01 + 0.05).astype(np.float32)
    code8, s2, off = nf4.double_quantize(a)
    dec = nf4.decode_scales(5000, code8=code8, s2=s2, offset=off)
    vals = np.array(sorted(set(nf4.dq_codebook().astype(np.float64).tolist())))
    half_gap = np.max(np.diff(vals)) / 2
    g = np.arange(5000) // 256
    bound = s2[g].astype(np.float64) * half_gap + 4 * np.spacing(np.float32(1.0)) * np.abs(a)
    assert np.all(np.abs(dec.astype(np.float64) - a) <= bound)


def test_codes_independent_of_double_quant_and_zero_block_stays_zero():
    rng = np.random.default_rng(9)
    w = (rng.standard_normal(64 * 40) * 0.02).astype(np.float32)
    w[64 * 3:64 * 4] = 0.0
    codes, absmax = nf4.quantize_nf4(w)
    payload, n = nf4.pack_codes(codes)
    code8, s2, off = nf4.double_quantize(absmax)
    a_dq = nf4.decode_scales(absmax.size, code8=code8, s2=s2, offset=off)
    w_dq = nf4.dequantize(payload, n, a_dq)
    w_plain = nf4.dequantize(payload, n, absmax)
    assert np.all(w_dq[64 * 3:64 * 4] == 0.0) and np.all(w_plain[64 * 3:64 * 4] == 0.0)
    # the scale error moves each weight by about C_j * delta_a
    C = np.array(nf4.NF4)[codes]
    delta = (a_dq.astype(np.float64) - absmax)[np.arange(w.size) // 64]
    assert np.all(np.abs((w_dq - w_plain) - C * delta) <= 2 * 2 ** -8 * np.abs(w_plain) + 1e-12)


def test_group_scale_is_the_max_over_every_position():
    """s2 is the absmax of the whole 256-group of centred scales (the page's
    blockwise absmax applied to the scales): placing the group's largest
    deviation at its first or at its last position must give that deviation
    as s2, and that scale must decode back within the error bound."""
    rng = np.random.default_rng(10)
    n1 = 256 * 3 + 40                       # ragged last group
    a = np.abs(rng.standard_normal(n1) * 0.002 + 0.05).astype(np.float32)
    a[255] = np.float32(0.9)                # last position of group 0
    a[256] = np.float32(0.8)                # first position of group 1
    a[n1 - 1] = np.float32(0.7)             # last position of the ragged group
    code8, s2, off = nf4.double_quantize(a)
    c = (a - off).astype(np.float32).astype(np.float64)
    for g in range(s2.size):
        grp = np.abs(c[g * 256:(g + 1) * 256])
        assert np.all(grp <= s2[g]) and np.any(grp == s2[g])
    dec = nf4.decode_scales(n1, code8=code8, s2=s2, offset=off).astype(np.float64)
    vals = np.array(sorted(set(nf4.dq_codebook().astype(np.float64).tolist())))
    half_gap = np.max(np.diff(vals)) / 2
    for i in (255, 256, n1 - 1):
        bound = float(s2[i // 256]) * half_gap + 4 * float(np.spacing(np.float32(1.0))) * a[i]
        assert abs(dec[i] - a[i]) <= bound


def test_exact_mean_subnormal_closed_forms():
    """Round to nearest even at the fp32 subnormal quantum 2^-149."""
    q = 2.0 ** -149
    assert nf4.exact_mean_f32(np.array([q, 0.0], np.float32)) == 0.0          # q/2: tie -> 0
    assert nf4.exact_mean_f32(np.array([3 * q, 0.0], np.float32)) == np.float32(2 * q)  # 1.5q -> 2q
    assert nf4.exact_mean_f32(np.array([q, q, q, 0.0], np.float32)) == np.float32(q)    # 0.75q -> q
    assert nf4.exact_mean_f32(np.array([5 * q, 0.0], np.float32)) == np.float32(2 * q)  # 2.5q -> 2q


def test_codebook_values_are_nearest_fp32_of_the_exact_ratio():
    """Each magnitude is the fp32 value nearest (num / den) as an exact
    rational, by enumeration of its fp32 neighbours."""
    table = nf4.dq_codebook()
    for t in range(1, 128):
        f = t.bit_length() - 1
        e, m = 6 - f, t - (1 << f)
        x = Fraction((1 << f) + 9 * (m + 1), (10 ** (e + 1)) * (1 << f))
        v = table[t]
        lo, hi = np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(2))
        d = abs(Fraction(float(v)) - x)
        assert d <= abs(Fraction(float(lo)) - x) and d <= abs(Fraction(float(hi)) - x), t


def test_double_quantize_exact_near_code_midpoints():
    """Centred scales placed on fp32 neighbours of s2 * (every midpoint of the
    8-bit codebook) get the exact-rational nearest code.  The values come in
    +-pairs so that the mean is exactly 0 and c = a."""
    table = nf4.dq_codebook()
    vals = sorted(set(float(v) for v in table if v > 0))
    pos_mids = [(Fraction(0) + Fraction(vals[0])) / 2]
    pos_mids += [(Fraction(vals[i]) + Fraction(vals[i + 1])) / 2 for i in range(len(vals) - 1)]
    D = np.float32(0.3)
    pts = []
    for mid in pos_mids:
        t = np.float32(float(Fraction(float(D)) * mid))
        for k in (-2, -1, 0, 1, 2):
            v = t
            for _ in range(abs(k)):
                v = np.nextafter(v, np.float32(np.inf if k > 0 else -np.inf))
            if 0 < v < D:
                pts.append(v)
    per = 127                                   # pairs per group after (D, -D)
    groups = []
    for i in range(0, len(pts), per):
        chunk = pts[i:i + per]
        g = [D, -D]
        for v in chunk:
            g += [v, -v]
        g += [np.float32(0.0)] * (256 - len(g))
        groups.append(g)
    a = np.array([v for g in groups for v in g], dtype=np.float32)
    code8, s2, off = nf4.double_quantize(a)
    assert off == 0.0 and np.all(s2 == D)
    for i in range(a.size):
        assert code8[i] == _brute_code8(a[i], D), i


def test_decode_rounds_the_product_before_adding_the_offset():
    """Rounding order of the scale decode ([P1] §"Double Quantization 压缩的是
    Scale": restore = decode + offset, every stored value fp32).  The reading
    taken is two fp32 roundings, a' = RN32(RN32(T8[q] * s2) + offset), with no
    fused multiply-add.  The values below separate it from a single rounding of
    the exact T8[q] * s2 + offset; the expected bits are worked out by hand:

      q = 0x43: sign 0, t = 67, f = 6, e = 0, m = 3, so
                |T8| = (2^6 + 9 * 4) / (10 * 2^6) = 100/640 = 5/32 exactly.
      s2 = 1 + 2^-23 (bits 0x3F800001).
      T8 * s2 = 5/32 + 5 * 2^-28 = 2^-3 * (1.25 + 2^-23 + 2^-25); the 2^-25
                term is below half an fp32 ulp of the product (2^-24 relative),
                so RN32(T8 * s2) = 5/32 + 2^-26.
      offset = -5/32 (bits 0xBE200000).
      two roundings: RN32(2^-26) = 2^-26               -> bits 0x32800000
      one rounding:  RN32(2^-26 + 2^-28) = 1.25 * 2^-26 -> bits 0x32A00000
    """
    code8 = np.array([0x43], dtype=np.uint8)
    s2 = np.array([0x3F800001], dtype=np.uint32).view(np.float32)
    offset = np.array([0xBE200000], dtype=np.uint32).view(np.float32)[0]
    got = nf4.decode_scales(1, code8=code8, s2=s2, offset=offset)
    assert got.dtype == np.float32
    assert int(got.view(np.uint32)[0]) == 0x32800000
    assert int(got.view(np.uint32)[0]) != 0x32A00000
    # the same decode further into a group: the group index picks s2[1]
    code8 = np.full(300, 0x43, dtype=np.uint8)
    s2 = np.array([0x3F800000, 0x3F800001], dtype=np.uint32).view(np.float32)
    got = nf4.decode_scales(300, code8=code8, s2=s2, offset=offset).view(np.uint32)
    assert np.all(got[:256] == 0) and np.all(got[256:] == 0x32800000)

"""NF4 encode / pack / unpack / double quantization / dequantize — CPU oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What each function follows, and what pins it (tests under ``tests/``):

* ``NF4`` — the 16-value table printed in [P1] §"从 NF4 索引打包成字节"
  (code block).  Pinned by the page's worked example and its printed
  reconstruction values.
* ``encode_block`` — [P1] §"NF4 保存的是索引而不是均匀整数值": absmax of a
  finite block, scale 1 for an all-zero block, nearest table value of w/a in
  Python doubles with ties to the smaller index.  Pinned by the page's
  examples and by an exact-rational brute force.
* ``quantize_nf4`` — the same rule vectorised over 64-element blocks of the
  row-major flattening.  Pinned against ``encode_block`` and brute force.
* ``pack_codes`` / ``unpack_codes`` — [P1] §"从 NF4 索引打包成字节": first code
  in the high nibble, odd tail padded with code 7, logical length kept;
  unpack checks the length and the padding code.  Pinned by bytes 79 3F.
* ``dq_codebook`` — the signed 8-bit dynamic codebook for scale codes.  The
  pages name it ([P1] §"Double Quantization 压缩的是 Scale") but print no
  table; this build defines it (see ``dq_codebook``).  Parity unpinned as to
  the table's values; its structural properties are pinned.
* ``exact_mean_f32`` — the global offset of double quantization: the mean of
  the first-level scales, computed exactly and rounded once to fp32.  Pinned
  by hand-computed ties and closed forms.
* ``double_quantize`` / ``decode_scales`` — [P1] §"Double Quantization 压缩的是
  Scale" and [P3] §3.2: subtract the mean, 256-blocks, fp32 second-level
  absmax, nearest 8-bit code; restore = decode + offset.  Pinned by
  invariants (equal group decodes to the offset; error bound; s2 the max
  over every group position) and by exact-rational brute force near every
  codebook midpoint.  The decode's two fp32 roundings (product, then sum)
  are a reading of "decode + offset" with fp32 storage, pinned by a
  hand-worked case whose one-rounding result differs.
* ``dequantize`` — [P1] §"NF4 保存的是索引而不是均匀整数值" (reconstruction
  a·C_j) and §"量化基座与可训练支路怎样相加" (computation in BF16): one
  rounding of the exact product to bf16.  Pinned by the page's printed
  reconstructions and the backward example's weights [0.5, -0.5].
* ``bit_budget`` — [P1] §"Double Quantization 压缩的是 Scale": 4.5 and
  4.126953125 bit per weight asymptotes.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

# [P1] §"从 NF4 索引打包成字节", the printed table (all entries are exact fp32).
NF4 = (
    -1.0, -0.6961928009986877, -0.5250730514526367,
    -0.39491748809814453, -0.28444138169288635, -0.18477343022823334,
    -0.09105003625154495, 0.0, 0.07958029955625534, 0.16093020141124725,
    0.24611230194568634, 0.33791524171829224, 0.44070982933044434,
    0.5626170039176941, 0.7229568362236023, 1.0,
)
_NF4 = np.array(NF4, dtype=np.float64)

BLOCKSIZE = 64        # first-level block ([P1] §"Double Quantization 压缩的是 Scale")
DQ_BLOCKSIZE = 256    # second-level block (same section)
PAD_CODE = 7          # odd-tail padding code ([P1] §"从 NF4 索引打包成字节")


class NonFiniteError(ValueError):
    """A block held a non-finite value, or a reconstruction was non-finite."""


class PaddingError(ValueError):
    """A packed payload disagrees with its logical length or padding code."""


# ----------------------------------------------------------------------------
# Encode
# ----------------------------------------------------------------------------
def encode_block(values):
    """One block, exactly as [P1] §"从 NF4 索引打包成字节" states the rule.

    Returns (codes, restored, scale).  Raises NonFiniteError on an empty or
    non-finite block and on a non-finite reconstruction.
    """
    values = [float(v) for v in values]
    if not values or any(not math.isfinite(v) for v in values):
        raise NonFiniteError("nonempty finite block required")
    amax = max(abs(v) for v in values)
    scale = amax if amax else 1.0
    codes = []
    for v in values:
        n = v / scale
        best = 0
        for j in range(1, 16):
            # strict '<' keeps the smaller index on an exact tie
            if abs(n - NF4[j]) < abs(n - NF4[best]):
                best = j
        codes.append(best)
    restored = [scale * NF4[j] for j in codes]
    if any(not math.isfinite(v) for v in restored):
        raise NonFiniteError("nonfinite reconstruction")
    return codes, restored, scale


def block_scales(w, blocksize: int = BLOCKSIZE):
    """The scale step alone: max|w| per block of the row-major flattening, or
    1.0 for an all-zero block, as fp32 (exact: it is an input magnitude)."""
    w = np.asarray(w, dtype=np.float32).ravel()
    P = w.size
    if P == 0:
        raise ValueError("empty tensor")
    n1 = -(-P // blocksize)
    full = (P // blocksize) * blocksize
    amax = np.empty(n1, dtype=np.float32)
    if full:
        amax[:P // blocksize] = np.max(np.abs(w[:full].reshape(-1, blocksize)), axis=1)
    if full < P:
        amax[-1] = np.max(np.abs(w[full:]))
    if not np.all(np.isfinite(amax)):
        raise NonFiniteError("nonempty finite block required")
    return np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)


def quantize_nf4(w, blocksize: int = BLOCKSIZE, chunk_blocks: int = 1 << 15):
    """Blockwise NF4 codes and fp32 scales for a flat array of weights.

    ``w``: the weights in row-major order (fp32 or bf16 values).  Blocks are
    consecutive runs of ``blocksize`` elements; the last one may be shorter.
    Returns (codes uint8[P], absmax float32[n1]) where absmax is the stored
    scale (1.0 for an all-zero block).
    """
    w = np.asarray(w, dtype=np.float64).ravel()
    P = w.size
    if P == 0:
        raise ValueError("empty tensor")
    if not np.all(np.isfinite(w)):
        raise NonFiniteError("nonempty finite block required")
    n1 = -(-P // blocksize)
    padded = np.zeros(n1 * blocksize, dtype=np.float64)
    padded[:P] = w            # |0| never raises a block's absmax
    blocks = padded.reshape(n1, blocksize)
    codes = np.empty((n1, blocksize), dtype=np.uint8)
    absmax = np.empty(n1, dtype=np.float64)
    for b0 in range(0, n1, chunk_blocks):
        blk = blocks[b0:b0 + chunk_blocks]
        amax = np.max(np.abs(blk), axis=1)
        scale = np.where(amax > 0, amax, 1.0)
        n = blk / scale[:, None]                       # Python-double division
        dist = np.abs(n[:, :, None] - _NF4[None, None, :])
        codes[b0:b0 + chunk_blocks] = np.argmin(dist, axis=2)  # first min = smaller index
        absmax[b0:b0 + chunk_blocks] = scale
    scale32 = absmax.astype(np.float32)
    assert np.all(scale32.astype(np.float64) == absmax), "scale must be an input magnitude"
    return codes.ravel()[:P], scale32


# ----------------------------------------------------------------------------
# Pack / unpack
# ----------------------------------------------------------------------------
def pack_codes(codes):
    """High nibble first, odd tail padded with code 7.  Returns (uint8[], length)."""
    codes = np.asarray(codes)
    if codes.size and (codes.min() < 0 or codes.max() > 15):
        raise ValueError("4-bit integer codes required")
    length = int(codes.size)
    c = codes.astype(np.uint8)
    if length % 2:
        c = np.concatenate([c, np.array([PAD_CODE], dtype=np.uint8)])
    payload = (c[0::2] << 4) | c[1::2]
    return payload.astype(np.uint8), length


def unpack_codes(payload, length: int):
    """Inverse of ``pack_codes`` with the page's two validity checks."""
    payload = np.asarray(payload, dtype=np.uint8)
    if length < 0 or payload.size != (length + 1) // 2:
        raise PaddingError("payload and logical length disagree")
    if length % 2 and (int(payload[-1]) & 15) != PAD_CODE:
        raise PaddingError("unexpected padding code")
    codes = np.empty(payload.size * 2, dtype=np.uint8)
    codes[0::2] = payload >> 4
    codes[1::2] = payload & 15
    return codes[:length]


# ----------------------------------------------------------------------------
# Double quantization
# ----------------------------------------------------------------------------
def dq_codebook():
    """256-entry signed dynamic 8-bit codebook for the scale codes (fp32).

    The pages require a signed dynamic 8-bit codebook that is not FP8 E4M3
    ([P1] §"Double Quantization 压缩的是 Scale") but print none.  This build
    defines one: byte u has sign u>>7 and magnitude index t = u & 127; t = 0
    is 0.0; otherwise with f = floor(log2 t), e = 6 - f, m = t - 2^f the
    magnitude is (2^f + 9(m+1)) / (10^(e+1) * 2^f), i.e. a decade exponent
    10^-e and a linear fraction in (0.1, 1], evaluated as a correctly rounded
    double division then rounded to fp32.
    """
    out = np.zeros(256, dtype=np.float32)
    for u in range(256):
        t = u & 127
        if t == 0:
            continue
        f = t.bit_length() - 1
        e = 6 - f
        m = t - (1 << f)
        num = (1 << f) + 9 * (m + 1)
        den = (10 ** (e + 1)) * (1 << f)
        mag = np.float32(num / den)
        out[u] = -mag if (u >> 7) else mag
    return out


def _round_rational_to_f32(p: int, q: int) -> np.float32:
    """Round the exact non-negative rational p/q to fp32, ties to even."""
    if q <= 0 or p < 0:
        raise ValueError("need p >= 0, q > 0")
    if p == 0:
        return np.float32(0.0)
    L = p.bit_length() - q.bit_length()
    ge = (p >= (q << L)) if L >= 0 else ((p << -L) >= q)
    fl = L if ge else L - 1                  # floor(log2(p/q))
    E = max(fl - 23, -149)                   # quantum 2^E: 24 bits, or subnormal
    num = p << -E if E < 0 else p
    den = q << E if E > 0 else q
    N, r = divmod(num, den)
    if 2 * r > den or (2 * r == den and (N & 1)):
        N += 1
    val = math.ldexp(N, E)
    if val > float(np.finfo(np.float32).max):
        return np.float32(np.inf)
    out = np.float32(val)
    assert float(out) == val
    return out


def exact_mean_f32(values) -> np.float32:
    """fp32 round-to-nearest-even of the exact mean of fp32 values.

    Every fp32 value is an integer multiple of 2^-149, so the sum is an
    exact integer in those units; one correctly rounded division follows.
    """
    v = np.asarray(values, dtype=np.float32)
    if v.size == 0:
        raise ValueError("empty")
    if not np.all(np.isfinite(v)):
        raise NonFiniteError("non-finite scale")
    m, e = np.frexp(v.astype(np.float64))           # v = m * 2^e, |m| in [0.5, 1)
    M = np.round(m * (1 << 24)).astype(np.int64)    # exact 24-bit integer mantissas
    assert np.all(M.astype(np.float64) == m * (1 << 24))
    # v = M * 2^(e-24) with e >= -148 for fp32, so in units of 2^-172 every
    # value is the integer M << (e - 24 + 172): the sum below is exact.
    total = 0
    for ex in np.unique(e):
        s = int(M[e == ex].sum())                   # |s| < 2^24 * n: exact in int64 for n < 2^39
        total += s << int(ex - 24 + 172)
    sign = 1
    if total < 0:
        sign, total = -1, -total
    r = _round_rational_to_f32(total, v.size << 172)
    return np.float32(sign * r)


def _nearest_sorted_fp64(x, values_sorted):
    """argmin_j |x - v_j| in fp64 over sorted values; ties -> smaller value."""
    d = np.abs(x[:, None] - values_sorted[None, :])
    return np.argmin(d, axis=1)


def double_quantize(absmax, blocksize: int = DQ_BLOCKSIZE, chunk: int = 1 << 16):
    """Quantize first-level scales: (code8 uint8[n1], s2 float32[n2], offset float32).

    [P1] §"Double Quantization 压缩的是 Scale": offset = mean of the
    first-level scales, subtract it, blockwise 8-bit quantization with block
    256 and an fp32 absmax per 256 (1.0 for an all-zero group), nearest code
    of c/s2 with ties to the smaller value.
    """
    a = np.asarray(absmax, dtype=np.float32).ravel()
    return double_quantize_centred(a, exact_mean_f32(a), blocksize, chunk)


def double_quantize_centred(absmax, offset, blocksize: int = DQ_BLOCKSIZE, chunk: int = 1 << 16):
    """The encoding half of ``double_quantize`` for a given offset (the mean
    of the whole tensor's scales): centre, then per group of 256 from the
    first element an fp32 absmax s2 and the nearest 8-bit code of c/s2."""
    a = np.asarray(absmax, dtype=np.float32).ravel()
    offset = np.float32(offset)
    n1 = a.size
    c = (a - offset).astype(np.float32)                   # fp32 subtraction, RN
    n2 = -(-n1 // blocksize)
    s2 = np.empty(n2, dtype=np.float32)
    for g in range(n2):
        mx = np.max(np.abs(c[g * blocksize:(g + 1) * blocksize]))
        s2[g] = mx if mx > 0 else np.float32(1.0)
    table = dq_codebook()
    distinct = np.unique(table.astype(np.float64))       # sorted; one zero
    code_of = {}
    for u in range(256):                                  # zero -> 0x00, else its byte
        code_of.setdefault(float(table[u]), u)
    sorted_codes = np.array([code_of[float(v)] for v in distinct], dtype=np.uint8)
    scale_el = np.repeat(s2.astype(np.float64), blocksize)[:n1]
    code8 = np.empty(n1, dtype=np.uint8)
    for i0 in range(0, n1, chunk):
        x = c[i0:i0 + chunk].astype(np.float64) / scale_el[i0:i0 + chunk]
        code8[i0:i0 + chunk] = sorted_codes[_nearest_sorted_fp64(x, distinct)]
    return code8, s2, np.float32(offset)


def decode_scales(n1, absmax=None, code8=None, s2=None, offset=None,
                  dq_blocksize: int = DQ_BLOCKSIZE):
    """Per-block decode scale a'.  Without DQ a' = absmax; with DQ
    a' = fp32(fp32(T8[q] * s2[g]) + offset), each step rounded (no fusion)."""
    if code8 is None:
        out = np.asarray(absmax, dtype=np.float32).ravel()
        assert out.size == n1
        return out
    table = dq_codebook()
    q = np.asarray(code8, dtype=np.uint8).ravel()
    assert q.size == n1
    g = np.arange(n1) // dq_blocksize
    t = (table[q] * np.asarray(s2, dtype=np.float32)[g]).astype(np.float32)
    out = (t + np.float32(offset)).astype(np.float32)
    return out


# ----------------------------------------------------------------------------
# Dequantize
# ----------------------------------------------------------------------------
def round_to_bf16(x):
    """Round fp64 values to bf16 (round to nearest, ties to even), as fp64."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    _, e = np.frexp(x[nz])                       # |x| in [2^(e-1), 2^e)
    quantum = np.ldexp(1.0, np.maximum(e, -125) - 8)   # 8 significant bits; subnormal 2^-133
    out[nz] = np.rint(x[nz] / quantum) * quantum        # exact scaling, np.rint = RNE
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    out[nz & (np.abs(out) > bf16_max)] = np.inf * np.sign(x[nz & (np.abs(out) > bf16_max)])
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


def bf16_bits(x):
    """uint16 bit patterns of bf16-representable fp64 values."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    assert np.all((f.astype(np.float64) == x) | np.isnan(x)), "not bf16-representable"
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def dequantize(packed, length: int, scales, blocksize: int = BLOCKSIZE):
    """Decode packed NF4 to bf16 values (returned as fp64 holding bf16 values).

    ``scales`` are the per-block decode scales a' (``decode_scales``).
    w_hat = RN_bf16(C_j * a'), the product exact in fp64 (24 x 24 bits).
    """
    codes = unpack_codes(packed, length)
    a = np.asarray(scales, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(a)):
        raise NonFiniteError("nonfinite reconstruction")
    per = a[np.arange(length) // blocksize]
    exact = _NF4[codes] * per
    return round_to_bf16(exact)


# ----------------------------------------------------------------------------
# Storage accounting
# ----------------------------------------------------------------------------
def bit_budget(P: int, double_quant: bool, blocksize: int = BLOCKSIZE,
               dq_blocksize: int = DQ_BLOCKSIZE) -> int:
    """Bits of payload + scale metadata for P weights ([P1] same section):
    8*ceil(P/2) + 32*n1 without DQ; 8*ceil(P/2) + 8*n1 + 32*n2 + 32 with DQ."""
    n1 = -(-P // blocksize)
    payload = 8 * ((P + 1) // 2)
    if not double_quant:
        return payload + 32 * n1
    n2 = -(-n1 // dq_blocksize)
    return payload + 8 * n1 + 32 * n2 + 32


def exact_fraction_nearest(x: Fraction, values) -> int:
    """Exact-rational argmin |x - v| over ``values``; ties -> smaller value.
    Used only as a brute-force pin (slow)."""
    best, bestd = None, None
    order = sorted(range(len(values)), key=lambda i: Fraction(float(values[i])))
    for i in order:
        d = abs(x - Fraction(float(values[i])))
        if bestd is None or d < bestd:
            best, bestd = i, d
    return best

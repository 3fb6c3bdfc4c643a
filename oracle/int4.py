"""Uniform signed INT4 blockwise quantization — CPU oracle (comparator type).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows [P2] "SFT（四）：QLoRA的4-bit量化与LoRA微调原理" §6 "先理解最普通的分块
量化": s = max|W| / 7, q_i = clip(round(w_i / s), -7, 7), w_hat_i = s q_i.
The page does not say how round() breaks ties; this oracle rounds half away
from zero (the usual school rule) and an all-zero block uses s = 1.
Pinned by the page's worked example W = [-1.20, -0.40, 0.10, 0.85] giving
q = [-7, -2, 1, 5] and W_hat ~ [-1.200, -0.343, 0.171, 0.857].
"""
from __future__ import annotations

import math


def int4_quantize_block(values):
    vals = [float(v) for v in values]
    if not vals or any(not math.isfinite(v) for v in vals):
        raise ValueError("nonempty finite block required")
    amax = max(abs(v) for v in vals)
    s = amax / 7.0 if amax else 1.0
    q = []
    for v in vals:
        t = v / s
        r = math.floor(abs(t) + 0.5) * (1 if t >= 0 else -1)
        q.append(max(-7, min(7, int(r))))
    return q, s


def int4_dequantize_block(q, s):
    return [s * v for v in q]


# ----------------------------------------------------------------------------
# Library storage format of the same quantizer (whole weights, vectorised)
# ----------------------------------------------------------------------------
# Readings of the page's formula for a stored format (the page shows the
# arithmetic only): blocks of 64 consecutive row-major elements, as NF4; the
# stored per-block scale is fp32, s = RN_fp32(amax / 7) with amax / 7 formed
# in fp64; q is decided on w / s in fp64 with the rule above (half away from
# zero, then clip to [-7, 7]); the code is q + 8 (1 .. 15), packed two per byte
# like NF4, and an odd tail is padded with code 8 (q = 0); the decoded weight
# is RN_bf16(q * s), the product exact.
INT4_PAD_CODE = 8


def int4_quantize(w, blocksize: int = 64):
    """Returns (codes uint8[numel], scales float32[n1]) of a flat weight."""
    import numpy as np
    x = np.asarray(w, dtype=np.float32).ravel().astype(np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("nonfinite input")
    n = x.size
    n1 = (n + blocksize - 1) // blocksize
    pad = n1 * blocksize - n
    xb = np.concatenate([x, np.zeros(pad)]).reshape(n1, blocksize)
    amax = np.max(np.abs(xb), axis=1)
    s = np.where(amax > 0, amax / 7.0, 1.0).astype(np.float32)
    t = xb / s.astype(np.float64)[:, None]
    r = np.floor(np.abs(t) + 0.5) * np.where(t >= 0, 1.0, -1.0)
    q = np.clip(r, -7, 7).astype(np.int64)
    codes = (q + 8).astype(np.uint8).ravel()[:n]
    return codes, s


def int4_dequantize(codes, scales, blocksize: int = 64):
    """RN_bf16((code - 8) * s) per element (fp64 holding bf16 values)."""
    import numpy as np
    from .nf4 import round_to_bf16
    c = np.asarray(codes, dtype=np.int64).ravel()
    s = np.asarray(scales, dtype=np.float32).astype(np.float64)
    per = s[np.arange(c.size) // blocksize]
    return round_to_bf16((c - 8) * per)

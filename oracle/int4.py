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

"""Merge / export of the trained layer — CPU oracle (fp64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows [P1] "QLoRA：冻结的 4-bit 权重怎样参与一次微调",
§"Merge 后还是不是训练时的函数": after training the layer's function is given by
the frozen W_hat together with the adapter.  It can be delivered (1) as
W_hat plus the separate adapter, (2) as one dense weight W_hat + c A B merged
in high precision, or (3) as that merged weight quantized again, which adds a
quantization step and is not the trained function in general.

``merge_exact`` is mode (2) in exact arithmetic (fp64; W_hat, A and B hold
bf16 values, so W_hat + c A B is formed to fp64 rounding).  The page fixes no
storage dtype for the merged weight; this library delivers it in the layer's
bf16 (``merge_bf16``: one round-to-nearest-even of the fp64 sum).  Mode (3)
is ``nf4.quantize_nf4`` applied to the delivered weight.

Pinned by the page's example (c A B = [0.03, 0.06], merged [0.53, -0.44],
output -0.35 for x = [1, 2]; re-quantization to codes [15, 1] with scale
0.53 is pinned in the NF4 tests), by X (W_hat + c A B) = lora_forward(X) for
random shapes, and by A = 0 leaving W_hat unchanged.
"""
from __future__ import annotations

import numpy as np

from .nf4 import round_to_bf16


def merge_exact(W_hat, A, B, c):
    """W_hat + c (A B) in fp64 (K x N)."""
    W_hat = np.asarray(W_hat, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    return W_hat + float(c) * (A @ B)


def merge_bf16(W_hat, A, B, c):
    """The delivered dense weight: RN_bf16(W_hat + c A B), as fp64 holding bf16 values."""
    return round_to_bf16(merge_exact(W_hat, A, B, c))

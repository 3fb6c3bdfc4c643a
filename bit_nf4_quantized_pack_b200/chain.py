"""A chain of frozen-NF4 + LoRA linear layers with a saved-activation policy.

Y_0 = X, Y_i = Y_{i-1} Ŵ_i + c_i (Y_{i-1} A_i) B_i, as in a stack of a decoder
layer's projections (the nonlinear parts of a real layer between them are not
part of this library).  The backward walks the layers in reverse; each layer's
input Y_{i-1} is kept, and its rank-r product Zc_i is either kept
(``policy="save"``) or recomputed inside the backward call
(``policy="recompute"``: M·r bf16 less per layer between the passes, at the
price of one rank-r contraction per layer; the page "SFT（四）：QLoRA的4-bit量化
与LoRA微调原理", §26.2 为什么开启 Gradient Checkpointing, states the same trade of
recomputation for stored activations).  Both policies give identical bits:
the recomputation uses the forward's kernel and split.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import linear_backward, linear_forward, new_status, status_sync
from ._lib import QLoRAError

__all__ = ["Layer", "LinearChain"]


@dataclass
class Layer:
    w: object          # NF4Weight of the K_i x N_i frozen base
    A: torch.Tensor    # K_i x r bf16
    B: torch.Tensor    # r x N_i bf16
    c: float


class LinearChain:
    def __init__(self, layers, policy: str = "save"):
        if policy not in ("save", "recompute"):
            raise ValueError("policy must be 'save' or 'recompute'")
        for a, b in zip(layers, layers[1:]):
            if a.w.shape[1] != b.w.shape[0]:
                raise ValueError("layer widths do not chain")
        self.layers = list(layers)
        self.policy = policy
        self._inputs = []
        self._zc = []

    def forward(self, X: torch.Tensor, status: torch.Tensor | None = None) -> torch.Tensor:
        own = status is None
        status = new_status(X.device) if own else status
        self._inputs, self._zc = [], []
        h = X
        for L in self.layers:
            self._inputs.append(h)
            h, zc = linear_forward(h, L.w, L.A, L.B, L.c, status=status)
            self._zc.append(zc if self.policy == "save" else None)
        if own:
            self._check(status, "forward")
        return h

    def backward(self, dY: torch.Tensor, status: torch.Tensor | None = None):
        """Returns (dX, [(dA_i, dB_i) for each layer])."""
        if not self._inputs:
            raise RuntimeError("backward before forward")
        own = status is None
        status = new_status(dY.device) if own else status
        grads = [None] * len(self.layers)
        g = dY
        for i in reversed(range(len(self.layers))):
            L = self.layers[i]
            g, dA, dB = linear_backward(g, self._inputs[i], self._zc[i], L.w, L.A, L.B, L.c,
                                        status=status)
            grads[i] = (dA, dB)
        if own:
            self._check(status, "backward")
        return g, grads

    @staticmethod
    def _check(status, where):
        code, mask = status_sync(status)
        if code != 0:
            raise QLoRAError(f"LinearChain.{where}: device status {code} (mask {mask})")

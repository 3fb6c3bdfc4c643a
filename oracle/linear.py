"""Frozen-base + LoRA linear layer, forward and backward — CPU oracle (fp64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows [P1] "QLoRA：冻结的 4-bit 权重怎样参与一次微调":
  §"量化基座与可训练支路怎样相加": X is M x K, W_hat is K x N, A is K x r,
      B is r x N, c = alpha / r; Y = X W_hat + c (X A) B.
  §"冻结权重为什么仍然需要输入梯度": Z = X A, Y = X W_hat + c Z B; with the
      output gradient G, dZ = c G B^T, and the input gradient flows through
      both branches: dX = G W_hat^T + dZ A^T; dA = X^T dZ; dB = c Z^T G.
      No gradient is formed for W_hat or its packed codes and scales.
Pinned by the worked example of §"一次完整反向与有限差分" (y = -0.35,
dX = [-0.7155, 0.594], dA = [-0.405, -0.81], dB = -0.675, B = 0 gives
dA = 0 and dB != 0) and by central finite differences of ``lora_forward``.
All arithmetic is fp64 on the given (bf16-valued) inputs; matrix products use
NumPy's matmul as a library primitive, with no blocking or reordering.
"""
from __future__ import annotations

import numpy as np


def lora_forward(X, W_hat, A, B, c):
    """Returns (Y, Z) with Z = X A and Y = X W_hat + c Z B, all fp64."""
    X = np.asarray(X, dtype=np.float64)
    W_hat = np.asarray(W_hat, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    Z = X @ A
    Y = X @ W_hat + float(c) * (Z @ B)
    return Y, Z


def lora_adapter_grads(G, X, A, B, c):
    """The trainable branch's part of the backward, which needs no W_hat:
    returns (dZ, dA, dB) with Z = X A, dZ = c G B^T, dA = X^T dZ, dB = c Z^T G,
    all fp64 ([P1] §"冻结权重为什么仍然需要输入梯度")."""
    G = np.asarray(G, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    c = float(c)
    Z = X @ A
    dZ = c * (G @ B.T)
    dA = X.T @ dZ
    dB = c * (Z.T @ G)
    return dZ, dA, dB


def lora_backward(G, X, W_hat, A, B, c):
    """Returns (dX, dA, dB) for the output gradient G, all fp64."""
    G = np.asarray(G, dtype=np.float64)
    W_hat = np.asarray(W_hat, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    dZ, dA, dB = lora_adapter_grads(G, X, A, B, c)
    dX = G @ W_hat.T + dZ @ A.T
    return dX, dA, dB

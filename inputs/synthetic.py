"""Seeded synthetic inputs for the five workload configurations.

This module only draws random tensors of the shapes, dtypes and value
distributions of the workloads; it holds none of the quantizer's or the
layer's arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle's
callers take their inputs from here.

Recipe: every tensor comes from NumPy ``default_rng(SeedSequence([seed,
cfg, tensor_id]))``; normals are drawn in fp64, multiplied by sigma, rounded
to fp32 and, for bf16 tensors, rounded to bf16 (nearest, ties to even).
Tensor ids: W=0, X=1, A=2, B=3, dY=4, outlier mask=5, plus 10*i for the i-th
matrix of a multi-matrix workload.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

W_ID, X_ID, A_ID, B_ID, DY_ID, MASK_ID = 0, 1, 2, 3, 4, 5


def rng_for(seed: int, cfg: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, cfg, tensor_id]))


def f32_to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (ties to even); returned as fp32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def bf16_bits(x_bf16_values: np.ndarray) -> np.ndarray:
    """uint16 storage of bf16-valued fp32 arrays."""
    x = np.ascontiguousarray(x_bf16_values, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def normal(seed, cfg, tid, shape, sigma, bf16=True) -> np.ndarray:
    g = rng_for(seed, cfg, tid)
    v = (g.standard_normal(size=shape) * sigma).astype(np.float32)
    return f32_to_bf16_values(v) if bf16 else v


@dataclass
class Linear:
    """One frozen-base LoRA linear: W is K x N (in x out), X is M x K."""
    name: str
    M: int
    K: int
    N: int
    W: np.ndarray | None = None
    X: np.ndarray | None = None
    A: np.ndarray | None = None
    B: np.ndarray | None = None
    dY: np.ndarray | None = None


@dataclass
class Workload:
    cfg: int
    name: str
    r: int
    alpha: float
    double_quant: bool
    w_dtype: str                     # "f32" or "bf16"
    linears: list = field(default_factory=list)
    backward: bool = True

    @property
    def c(self) -> float:
        return float(np.float32(self.alpha / self.r))


def _outliers(W, seed, cfg, tid, frac, value):
    g = rng_for(seed, cfg, tid)
    mask = g.random(W.shape) < frac
    sign = np.where(g.random(W.shape) < 0.5, -1.0, 1.0).astype(np.float32)
    W = W.copy()
    W[mask] = (value * sign[mask]).astype(np.float32)
    return W


def make_linear(cfg, i, name, M, K, N, w_sigma, r, *, seed=0, w_bf16=True,
                outlier_frac=0.0, outlier_value=0.0, with_x=True, with_dy=True,
                lora_sigma=0.01):
    base = 10 * i
    lin = Linear(name=name, M=M, K=K, N=N)
    W = normal(seed, cfg, base + W_ID, (K, N), w_sigma, bf16=False)
    if outlier_frac:
        W = _outliers(W, seed, cfg, base + MASK_ID, outlier_frac, outlier_value)
    lin.W = f32_to_bf16_values(W) if w_bf16 else W
    if with_x:
        lin.X = normal(seed, cfg, base + X_ID, (M, K), 1.0)
    lin.A = normal(seed, cfg, base + A_ID, (K, r), lora_sigma)
    lin.B = normal(seed, cfg, base + B_ID, (r, N), lora_sigma)
    if with_dy:
        lin.dY = normal(seed, cfg, base + DY_ID, (M, N), 1.0)
    return lin


def config1(seed=0) -> Workload:
    """Tiny: W 256x256 fp32 ~N(0,0.02) with +-0.3 every 97th entry and one
    all-zero 64-block; X 16x256; r=8, alpha=16; no double quant."""
    wl = Workload(cfg=1, name="tiny-256x256-m16-r8", r=8, alpha=16.0,
                  double_quant=False, w_dtype="f32")
    lin = make_linear(1, 0, "tiny", 16, 256, 256, 0.02, 8, seed=seed, w_bf16=False)
    flat = lin.W.reshape(-1).copy()
    idx = np.arange(flat.size)
    hit = (idx % 97) == 96
    flat[hit] = np.where((idx[hit] // 97) % 2 == 0, 0.3, -0.3).astype(np.float32)
    flat[320:384] = 0.0
    lin.W = flat.reshape(256, 256)
    wl.linears.append(lin)
    return wl


def config2(seed=0, M=4096) -> Workload:
    """One 7B-shaped projection: W 4096x4096 bf16 ~N(0,0.02), DQ; X M x 4096."""
    wl = Workload(cfg=2, name="proj-4096x4096-m4096-r16", r=16, alpha=32.0,
                  double_quant=True, w_dtype="bf16")
    wl.linears.append(make_linear(2, 0, "proj", M, 4096, 4096, 0.02, 16, seed=seed))
    return wl


def config3(seed=0, Ms=(1, 4, 16)) -> Workload:
    """Decode-style GEMV: W 4096x11008 and 11008x4096, DQ; M in {1,4,16}; fwd only."""
    wl = Workload(cfg=3, name="gemv-4096x11008", r=16, alpha=32.0,
                  double_quant=True, w_dtype="bf16", backward=False)
    shapes = [("up", 4096, 11008), ("down", 11008, 4096)]
    for i, (nm, K, N) in enumerate(shapes):
        lin = make_linear(3, i, nm, max(Ms), K, N, 0.02, 16, seed=seed, with_dy=False)
        wl.linears.append(lin)
    return wl


LAYER7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
           ("gate", 4096, 11008), ("up", 4096, 11008), ("down", 11008, 4096)]


def config4(seed=0, M=4096, with_data=True) -> Workload:
    """7B decoder-layer linear set, 0.1% outliers at 10 sigma; r=64, alpha=16."""
    wl = Workload(cfg=4, name="layer7b-7linears-m4096-r64", r=64, alpha=16.0,
                  double_quant=True, w_dtype="bf16")
    for i, (nm, K, N) in enumerate(LAYER7B):
        wl.linears.append(make_linear(4, i, nm, M, K, N, 0.02, 64, seed=seed,
                                      outlier_frac=0.001, outlier_value=0.2,
                                      with_x=with_data, with_dy=with_data))
    return wl


def config5(seed=0, M=4096, with_data=True) -> Workload:
    """65B MLP slice: W 8192x22016 and 22016x8192 ~N(0,0.015); r=64, alpha=16."""
    wl = Workload(cfg=5, name="mlp65b-8192x22016-m4096-r64", r=64, alpha=16.0,
                  double_quant=True, w_dtype="bf16")
    for i, (nm, K, N) in enumerate([("up", 8192, 22016), ("down", 22016, 8192)]):
        wl.linears.append(make_linear(5, i, nm, M, K, N, 0.015, 64, seed=seed,
                                      with_x=with_data, with_dy=with_data))
    return wl


def random_case(seed, M, K, N, r, *, w_sigma=0.02, w_bf16=True, lora_sigma=0.01):
    """A small seeded case for parity tests (cfg id 100)."""
    return make_linear(100 + seed, 0, "case", M, K, N, w_sigma, r, seed=seed,
                       w_bf16=w_bf16, lora_sigma=lora_sigma)

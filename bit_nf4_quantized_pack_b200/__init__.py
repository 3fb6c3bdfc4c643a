"""NF4 frozen-base LoRA linear layer for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/qlora_nf4.h``: PyTorch is used
for device memory and the current CUDA stream only; every step of the
computation runs in the library's CUDA kernels.  The calls mirror the C
entry points:

    quantize(W, double_quant)            -> NF4Weight     (qlora_nf4_quantize)
    dequantize(w)                        -> bf16 K x N    (qlora_nf4_dequantize)
    linear_forward(X, w, A, B, c)        -> (Y, Zc)       (qlora_linear_fwd)
    linear_backward(dY, X, Zc, w, A, B, c) -> (dX, dA, dB) (qlora_linear_bwd)

Page "QLoRA：冻结的 4-bit 权重怎样参与一次微调" defines the method (see the
header for the section of each call).
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import NF4StateC, QLoRAError, check, lib

__all__ = ["NF4Weight", "quantize", "dequantize", "merge", "merge_requantize",
           "quantize_shard_begin", "quantize_shard_end", "shard_workspace_size",
           "linear_forward", "linear_backward",
           "status_sync", "status_clear", "new_status", "QLoRAError", "lib"]

BLOCKSIZE = 64
DQ_BLOCKSIZE = 256


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def n1_of(numel: int) -> int:
    return int(lib.qlora_nf4_n1(numel))


def n2_of(numel: int) -> int:
    return int(lib.qlora_nf4_n2(numel))


@dataclass
class NF4Weight:
    """Quantized state of a K x N weight (the caller-owned buffers of
    ``qlora_nf4_state``)."""
    shape: tuple
    double_quant: bool
    packed: torch.Tensor
    absmax: torch.Tensor | None = None
    code8: torch.Tensor | None = None
    s2: torch.Tensor | None = None
    offset: torch.Tensor | None = None
    codebook: int = 0      # 0: NF4, 1: uniform INT4 (absmax then holds s = amax / 7)

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= int(s)
        return n

    def cstruct(self) -> NF4StateC:
        st = NF4StateC()
        st.numel = self.numel
        st.blocksize = BLOCKSIZE
        st.double_quant = 1 if self.double_quant else 0
        st.dq_blocksize = DQ_BLOCKSIZE
        st.codebook = int(self.codebook)
        st.packed = self.packed.data_ptr()
        st.absmax = self.absmax.data_ptr() if self.absmax is not None else None
        st.code8 = self.code8.data_ptr() if self.code8 is not None else None
        st.s2 = self.s2.data_ptr() if self.s2 is not None else None
        st.offset = self.offset.data_ptr() if self.offset is not None else None
        return st

    @staticmethod
    def empty(shape, double_quant: bool, device="cuda", codebook: int = 0) -> "NF4Weight":
        numel = 1
        for s in shape:
            numel *= int(s)
        n1, n2 = n1_of(numel), n2_of(numel)
        u8, f32 = torch.uint8, torch.float32
        if codebook and double_quant:
            raise ValueError("the INT4 codebook has no double quantization")
        w = NF4Weight(tuple(int(s) for s in shape), bool(double_quant),
                      torch.empty((numel + 1) // 2, dtype=u8, device=device), codebook=int(codebook))
        if double_quant:
            w.code8 = torch.empty(n1, dtype=u8, device=device)
            w.s2 = torch.empty(n2, dtype=f32, device=device)
            w.offset = torch.empty(1, dtype=f32, device=device)
        else:
            w.absmax = torch.empty(n1, dtype=f32, device=device)
        return w


def new_status(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def status_sync(status: torch.Tensor):
    """(first error code or 0, raw bit mask); synchronizes the current stream."""
    mask = C.c_int32(0)
    code = lib.qlora_status_sync(_ptr(status), _stream(), C.byref(mask))
    return int(code), int(mask.value)


def status_clear(status: torch.Tensor) -> None:
    check(lib.qlora_status_clear(_ptr(status), _stream()), "qlora_status_clear")


class _WorkspaceCache:
    """Reuses one device buffer per (purpose, device, current stream) so
    repeated calls do not allocate; grows when a larger workspace is needed.
    Keyed by stream as well: calls in flight on two streams never share a
    buffer, and each buffer is allocated and used in one stream's order.
    At most ``limit`` buffers are kept (the least recently used is dropped;
    the caching allocator reuses its memory in its own stream's order).

    CUDA graphs: a captured launch keeps the raw pointer of its workspace.
    While the current stream is capturing, ``get`` never allocates, grows or
    drops a buffer (a call that needs more than the cached buffer raises: pass
    ``workspace=`` explicitly, or make the same call once before capturing),
    and every buffer handed out during a capture stays referenced for the life
    of the process, so a later, larger call that replaces it cannot hand its
    memory to another tensor while a graph still writes into it."""

    def __init__(self, limit: int = 16):
        self._bufs = {}
        self._limit = limit
        self._captured = []

    def get(self, key, nbytes, device):
        if nbytes == 0:
            return None
        stream = torch.cuda.current_stream(device)
        key = (*key, stream.cuda_stream)
        buf = self._bufs.get(key)
        if torch.cuda.is_current_stream_capturing():
            if buf is None or buf.numel() < nbytes or buf.device != torch.device(device):
                raise RuntimeError(
                    "no workspace of the needed size is cached for this stream while it is "
                    "capturing a CUDA graph: pass workspace= or run the call once before capture")
            if not any(b is buf for b in self._captured):
                self._captured.append(buf)
            return buf
        self._bufs.pop(key, None)
        if buf is None or buf.numel() < nbytes or buf.device != torch.device(device):
            buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        self._bufs[key] = buf                    # most recently used last
        while len(self._bufs) > self._limit:
            self._bufs.pop(next(iter(self._bufs)))
        return buf


_ws = _WorkspaceCache()


def _finish(status, own_status, where):
    if own_status:
        code, _ = status_sync(status)
        check(code, where)


def quantize(W: torch.Tensor, double_quant: bool = True, *, out: NF4Weight | None = None,
             status: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
             codebook: str = "nf4") -> NF4Weight:
    """Blockwise 4-bit quantization of a contiguous bf16 or fp32 CUDA tensor:
    codebook "nf4" (optionally double-quantized) or "int4" (uniform signed)."""
    if codebook not in ("nf4", "int4"):
        raise ValueError("codebook must be 'nf4' or 'int4'")
    cb = 1 if codebook == "int4" else 0
    if cb:
        double_quant = False
    if W.dtype == torch.bfloat16:
        dt = _lib.QLORA_DTYPE_BF16
    elif W.dtype == torch.float32:
        dt = _lib.QLORA_DTYPE_F32
    else:
        raise TypeError("W must be bfloat16 or float32")
    if not W.is_contiguous():
        raise ValueError("W must be contiguous")
    w = out if out is not None else NF4Weight.empty(W.shape, double_quant, W.device, codebook=cb)
    if w.codebook != cb:
        raise ValueError("out has another codebook")
    st = w.cstruct()
    need = int(lib.qlora_nf4_quantize_workspace_size(w.numel, st.double_quant))
    ws = workspace if workspace is not None else _ws.get(("q", W.device), need, W.device)
    own = status is None
    status = new_status(W.device) if own else status
    check(lib.qlora_nf4_quantize(_ptr(W), dt, C.byref(st), _ptr(ws),
                                 ws.numel() if ws is not None else 0, _ptr(status), _stream()),
          "qlora_nf4_quantize")
    _finish(status, own, "qlora_nf4_quantize")
    return w


def shard_workspace_size(numel: int, block_begin: int, block_end: int, double_quant: bool) -> int:
    return int(lib.qlora_nf4_quantize_shard_workspace_size(numel, block_begin, block_end,
                                                           1 if double_quant else 0))


def _dtype_code(W):
    if W.dtype == torch.bfloat16:
        return _lib.QLORA_DTYPE_BF16
    if W.dtype == torch.float32:
        return _lib.QLORA_DTYPE_F32
    raise TypeError("W must be bfloat16 or float32")


def quantize_shard_begin(W_shard: torch.Tensor, w: NF4Weight, block_begin: int, block_end: int, *,
                         workspace: torch.Tensor | None, status: torch.Tensor | None = None) -> None:
    """Phase 1 of a sharded quantization (qlora_nf4_quantize_shard_begin):
    encode 64-blocks [block_begin, block_end) of the weight `w` describes;
    W_shard holds exactly those elements (contiguous)."""
    if not W_shard.is_contiguous():
        raise ValueError("W_shard must be contiguous")
    st = w.cstruct()
    dev = w.packed.device
    own = status is None
    status = new_status(dev) if own else status
    check(lib.qlora_nf4_quantize_shard_begin(
        _ptr(W_shard) if W_shard.numel() else None, _dtype_code(W_shard), C.byref(st), block_begin,
        block_end, _ptr(workspace), workspace.numel() if workspace is not None else 0,
        _ptr(status), _stream()), "qlora_nf4_quantize_shard_begin")
    _finish(status, own, "qlora_nf4_quantize_shard_begin")


def quantize_shard_end(w: NF4Weight, block_begin: int, block_end: int, *,
                       workspace: torch.Tensor | None, status: torch.Tensor | None = None) -> None:
    """Phase 2 (qlora_nf4_quantize_shard_end): the workspace's first 2048 bytes
    must hold the exponent bins summed over every shard."""
    st = w.cstruct()
    dev = w.packed.device
    own = status is None
    status = new_status(dev) if own else status
    check(lib.qlora_nf4_quantize_shard_end(
        C.byref(st), block_begin, block_end, _ptr(workspace),
        workspace.numel() if workspace is not None else 0, _ptr(status), _stream()),
        "qlora_nf4_quantize_shard_end")
    _finish(status, own, "qlora_nf4_quantize_shard_end")


def dequantize(w: NF4Weight, *, out: torch.Tensor | None = None,
               status: torch.Tensor | None = None) -> torch.Tensor:
    dev = w.packed.device
    out = out if out is not None else torch.empty(w.shape, dtype=torch.bfloat16, device=dev)
    st = w.cstruct()
    own = status is None
    status = new_status(dev) if own else status
    check(lib.qlora_nf4_dequantize(C.byref(st), _ptr(out), _ptr(status), _stream()),
          "qlora_nf4_dequantize")
    _finish(status, own, "qlora_nf4_dequantize")
    return out


def merge(w: NF4Weight, A, B, c: float, *, out: torch.Tensor | None = None,
          status: torch.Tensor | None = None) -> torch.Tensor:
    """The merged dense weight RN_bf16(Ŵ + c·A·B) (K x N bf16)."""
    for t, n in ((A, "A"), (B, "B")):
        _bf16(t, n)
    K, N = w.shape
    r = A.shape[1]
    if A.shape[0] != K or tuple(B.shape) != (r, N):
        raise ValueError("shape mismatch")
    dev = w.packed.device
    out = out if out is not None else torch.empty((K, N), dtype=torch.bfloat16, device=dev)
    _bf16(out, "out")
    st = w.cstruct()
    own = status is None
    status = new_status(dev) if own else status
    check(lib.qlora_nf4_merge(K, N, r, C.byref(st), _ptr(A), _ptr(B), float(c), _ptr(out),
                              _ptr(status), _stream()), "qlora_nf4_merge")
    _finish(status, own, "qlora_nf4_merge")
    return out


def merge_requantize(w: NF4Weight, A, B, c: float, double_quant: bool = True, *,
                     status: torch.Tensor | None = None) -> NF4Weight:
    """The merged weight quantized again to NF4 (a new quantization step)."""
    return quantize(merge(w, A, B, c, status=status), double_quant=double_quant, status=status)


def _bf16(t, name):
    if t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda:
        raise TypeError(f"{name} must be a contiguous CUDA bfloat16 tensor")


def linear_forward(X, w: NF4Weight, A, B, c: float, *, Y=None, Zc=None, status=None,
                   workspace=None):
    """Y = X·Ŵ + c·(X·A)·B with Ŵ decoded on the fly; returns (Y, Zc)."""
    for t, n in ((X, "X"), (A, "A"), (B, "B")):
        _bf16(t, n)
    M, K = X.shape
    Kw, N = w.shape
    r = A.shape[1]
    if Kw != K or A.shape[0] != K or tuple(B.shape) != (r, N):
        raise ValueError("shape mismatch")
    dev = X.device
    Y = Y if Y is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    Zc = Zc if Zc is not None else torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    need = int(lib.qlora_linear_fwd_workspace_size(M, K, N, r))
    ws = workspace if workspace is not None else _ws.get(("f", dev), need, dev)
    st = w.cstruct()
    own = status is None
    status = new_status(dev) if own else status
    check(lib.qlora_linear_fwd(M, K, N, r, _ptr(X), C.byref(st), _ptr(A), _ptr(B), float(c),
                               _ptr(Y), _ptr(Zc), _ptr(ws), ws.numel() if ws is not None else 0,
                               _ptr(status), _stream()), "qlora_linear_fwd")
    _finish(status, own, "qlora_linear_fwd")
    return Y, Zc


def linear_backward(dY, X, Zc, w: NF4Weight, A, B, c: float, *, dX=None, dA=None, dB=None,
                    status=None, workspace=None):
    """dX = dY·Ŵᵀ + c·(dY·Bᵀ)·Aᵀ, dA = Xᵀ·(c·dY·Bᵀ), dB = Zcᵀ·dY; returns (dX, dA, dB).
    Zc=None recomputes bf16(c·X·A) inside the call (bit-identical to the forward's)."""
    for t, n in ((dY, "dY"), (X, "X"), (A, "A"), (B, "B")):
        _bf16(t, n)
    if Zc is not None:
        _bf16(Zc, "Zc")
    M, K = X.shape
    N = dY.shape[1]
    r = A.shape[1]
    dev = X.device
    dX = dX if dX is not None else torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty((K, r), dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty((r, N), dtype=torch.float32, device=dev)
    need = int(lib.qlora_linear_bwd_workspace_size(M, K, N, r))
    ws = workspace if workspace is not None else _ws.get(("b", dev), need, dev)
    st = w.cstruct()
    own = status is None
    status = new_status(dev) if own else status
    check(lib.qlora_linear_bwd(M, K, N, r, _ptr(dY), _ptr(X), _ptr(Zc) if Zc is not None else None,
                               C.byref(st), _ptr(A),
                               _ptr(B), float(c), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(ws),
                               ws.numel() if ws is not None else 0, _ptr(status), _stream()),
          "qlora_linear_bwd")
    _finish(status, own, "qlora_linear_bwd")
    return dX, dA, dB

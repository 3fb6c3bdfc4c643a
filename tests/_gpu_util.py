"""Helpers shared by the GPU parity tests (oracle side and device side kept
apart: the oracle only ever sees NumPy inputs from the seeded generators)."""
import numpy as np
import torch

from oracle import nf4


def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_dev(x, dtype=torch.bfloat16):
    """NumPy fp32 array (bf16-valued for bf16 tensors) -> contiguous CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev()).to(dtype).contiguous()


def to_np(t):
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def bf16_bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().astype(np.uint16)


def rel_fro(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


class OracleWeight:
    """The oracle's own quantization of a weight, from the same NumPy input."""

    def __init__(self, W, double_quant):
        w = np.asarray(W, dtype=np.float32).ravel()
        self.shape = np.asarray(W).shape
        self.codes, self.absmax = nf4.quantize_nf4(w)
        self.packed, self.length = nf4.pack_codes(self.codes)
        self.dq = double_quant
        if double_quant:
            self.code8, self.s2, self.offset = nf4.double_quantize(self.absmax)
            self.scales = nf4.decode_scales(self.absmax.size, code8=self.code8, s2=self.s2,
                                            offset=self.offset)
        else:
            self.scales = self.absmax
        self._what = None

    @property
    def w_hat(self):
        if self._what is None:
            self._what = nf4.dequantize(self.packed, self.length, self.scales).reshape(self.shape)
        return self._what


def assert_state_equal(w_gpu, ow: OracleWeight):
    assert np.array_equal(w_gpu.packed.cpu().numpy(), ow.packed), "packed bytes differ"
    if ow.dq:
        assert np.array_equal(w_gpu.code8.cpu().numpy(), ow.code8), "scale codes differ"
        assert np.array_equal(w_gpu.s2.cpu().numpy().view(np.uint32), ow.s2.view(np.uint32)), "s2 differs"
        assert w_gpu.offset.cpu().numpy().view(np.uint32)[0] == np.float32(ow.offset).view(np.uint32), \
            "offset differs"
    else:
        assert np.array_equal(w_gpu.absmax.cpu().numpy().view(np.uint32), ow.absmax.view(np.uint32)), \
            "absmax differs"


# Element-wise bounds on top of the whole-matrix relative Frobenius error: a
# handful of wrong outputs, or one wrong 64-column block in one row, moves the
# whole-matrix norm of a large output by far less than 5e-3, but not the error
# of its row or of its tile.
FRO_TOL = 5e-3
ROW_TOL = 1e-2
TILE_TOL = 2e-2


def close_report(got, ref, tile=128, row_elems=256):
    """Relative errors of `got` against `ref`: whole matrix (Frobenius), worst
    row, worst tile x tile block.  A "row" is a group of consecutive rows with
    at least `row_elems` elements (one row of a wide matrix; several rows of a
    narrow one such as dA, K x r, where a single element's relative error says
    nothing).  A row or tile whose reference norm is tiny is measured against a
    tenth of the typical row or tile norm instead."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.ndim == 1:
        got, ref = got[None, :], ref[None, :]
    assert got.shape == ref.shape, (got.shape, ref.shape)
    diff = got - ref
    total = np.linalg.norm(ref)
    out = {"fro": float(np.linalg.norm(diff) / (total if total > 0 else 1.0))}
    R, C = ref.shape
    rb = max(1, -(-row_elems // C))             # rows per group
    Rg = -(-R // rb)

    def row_norms(a):
        p = np.zeros((Rg * rb, C))
        p[:R] = a
        return np.sqrt((p.reshape(Rg, rb * C) ** 2).sum(axis=1))

    row_rms = total / np.sqrt(Rg)
    rn, dn = row_norms(ref), row_norms(diff)
    out["row"] = float(np.max(dn / np.maximum(rn, max(0.1 * row_rms, 1e-300))))
    tr, tc = min(tile, R), min(tile, C)
    Rp, Cp = -(-R // tr) * tr, -(-C // tc) * tc

    def blocks(a):
        p = np.zeros((Rp, Cp))
        p[:R, :C] = a
        return np.sqrt((p.reshape(Rp // tr, tr, Cp // tc, tc) ** 2).sum(axis=(1, 3)))

    tn, td = blocks(ref), blocks(diff)
    tile_rms = total / np.sqrt(tn.size)
    out["tile"] = float(np.max(td / np.maximum(tn, max(0.1 * tile_rms, 1e-300))))
    return out


def assert_close(name, got, ref, fro=FRO_TOL, row=ROW_TOL, tile_tol=TILE_TOL):
    rep = close_report(got, ref)
    assert rep["fro"] <= fro and rep["row"] <= row and rep["tile"] <= tile_tol, (name, rep)
    return rep

"""GPU parity of qlora_linear_fwd / qlora_linear_bwd against the fp64 oracle.

Bar: for Y, Zc, dX, dA, dB (each against the oracle's fp64 result on the
oracle's own dequantized weight) a whole-matrix relative Frobenius error <=
5e-3, and the worst row's and worst 128 x 128 tile's relative error within the
bounds of tests/_gpu_util.py; exact special cases where the arithmetic makes
them exact.
"""
import numpy as np
import pytest
import torch

from inputs import synthetic as S
from oracle.linear import lora_adapter_grads, lora_backward, lora_forward
from tests._gpu_util import OracleWeight, assert_close, close_report, rel_fro, to_dev, to_np

pytestmark = pytest.mark.gpu
TOL = 5e-3


def _q():
    import bit_nf4_quantized_pack_b200 as q
    return q


def run_case(lin, r, c, dq, *, backward=True, w_dtype=torch.bfloat16):
    q = _q()
    X, W, A, B = lin.X, lin.W, lin.A, lin.B
    wq = q.quantize(to_dev(W, w_dtype), double_quant=dq)
    Xt, At, Bt = to_dev(X), to_dev(A), to_dev(B)
    Y, Zc = q.linear_forward(Xt, wq, At, Bt, c)
    ow = OracleWeight(W, dq)
    Yr, Zr = lora_forward(X, ow.w_hat, A, B, c)
    out = {"Y": assert_close("Y", to_np(Y), Yr)["fro"],
           "Zc": assert_close("Zc", to_np(Zc), c * Zr)["fro"]}
    if backward:
        G = lin.dY
        dX, dA, dB = q.linear_backward(to_dev(G), Xt, Zc, wq, At, Bt, c)
        dXr, dAr, dBr = lora_backward(G, X, ow.w_hat, A, B, c)
        out.update(dX=assert_close("dX", to_np(dX), dXr)["fro"],
                   dA=assert_close("dA", to_np(dA), dAr)["fro"],
                   dB=assert_close("dB", to_np(dB), dBr)["fro"])
        # the recompute policy (no saved Zc) gives the same bits
        dX2, dA2, dB2 = q.linear_backward(to_dev(G), Xt, None, wq, At, Bt, c)
        for a_, b_ in zip((dX, dA, dB), (dX2, dA2, dB2)):
            assert torch.equal(a_, b_)
    return out


CASES = [
    # (M, K, N, r, dq)  — several tiles in every dimension plus ragged edges
    (200, 320, 384, 16, True),
    (129, 256, 512, 8, False),
    (300, 512, 192, 64, True),
    (257, 1024, 768, 32, True),
    (17, 128, 256, 16, False),
    (128, 64, 64, 8, True),
]


@pytest.mark.parametrize("M,K,N,r,dq", CASES)
def test_fwd_bwd_parity(M, K, N, r, dq):
    lin = S.random_case(M + K + N + r, M, K, N, r)
    lin.dY = S.normal(7, M, 4, (M, N), 1.0)
    errs = run_case(lin, r, 32.0 / r, dq)
    for k, v in errs.items():
        assert v <= TOL, (k, v, errs)


ODD_RANK_CASES = [
    # (M, K, N, r): ranks that are not multiples of 8, zero-padded inside the
    # workspace; tensor-core path (M > 16) and GEMV (M <= 16), fwd and bwd
    (200, 256, 320, 1),
    (129, 320, 256, 3),
    (300, 512, 192, 12),
    (160, 384, 512, 40),
    (1, 256, 320, 1),
    (4, 320, 448, 3),
    (9, 512, 384, 12),
    (16, 576, 256, 40),
]


@pytest.mark.parametrize("M,K,N,r", ODD_RANK_CASES)
def test_ranks_not_multiple_of_8(M, K, N, r):
    lin = S.random_case(3000 + M + K + N + r, M, K, N, r)
    lin.dY = S.normal(13, M + r, 4, (M, N), 1.0)
    errs = run_case(lin, r, 16.0 / r, True)
    for k, v in errs.items():
        assert v <= TOL, (k, v, errs)


@pytest.mark.parametrize("M", [1, 2, 4, 5, 8, 16])
def test_gemv_parity(M):
    lin = S.random_case(100 + M, M, 640, 576, 16)
    errs = run_case(lin, 16, 2.0, True, backward=False)
    for k, v in errs.items():
        assert v <= TOL, (k, v, errs)


MULTI_WAVE_CASES = [
    # more 512 x 128 tiles than SMs, the last wave partial: the persistent
    # CTAs take a second tile (forward in the first case, dX in the second)
    (2048, 1024, 8192, 16, True),
    (2048, 8192, 1024, 16, False),
]


@pytest.mark.parametrize("M,K,N,r,dq", MULTI_WAVE_CASES)
def test_multi_wave_parity(M, K, N, r, dq):
    lin = S.random_case(M + 3 * K + N, M, K, N, r)
    lin.dY = S.normal(11, M, 4, (M, N), 1.0)
    errs = run_case(lin, r, 32.0 / r, dq)
    for k, v in errs.items():
        assert v <= TOL, (k, v, errs)


def test_forward_deterministic():
    """Every sum has a fixed order: repeated launches give the same bits."""
    q = _q()
    lin = S.random_case(42, 2048, 1024, 8192, 16)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    Xt, At, Bt = to_dev(lin.X), to_dev(lin.A), to_dev(lin.B)
    Y1, _ = q.linear_forward(Xt, wq, At, Bt, 2.0)
    for _ in range(3):
        Y2, _ = q.linear_forward(Xt, wq, At, Bt, 2.0)
        assert torch.equal(Y1, Y2)


def test_backward_streams_and_graph_capture():
    """The backward runs dA and dB on a library stream beside dX and joins it
    back into the caller's stream.  Bits must not depend on that: the same
    call on the default stream, on another torch stream, repeated, and
    captured in a CUDA graph and replayed gives identical dX, dA and dB."""
    q = _q()
    M, K, N, r = 1536, 1024, 2048, 16   # dX: 3 x 8 = 24 tiles; dA/dB: several clusters
    lin = S.random_case(55, M, K, N, r)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    Xt, At, Bt = to_dev(lin.X), to_dev(lin.A), to_dev(lin.B)
    G = to_dev(S.normal(9, M, 4, (M, N), 1.0))
    _, Zc = q.linear_forward(Xt, wq, At, Bt, 2.0)
    ref = q.linear_backward(G, Xt, Zc, wq, At, Bt, 2.0)
    torch.cuda.synchronize()
    for _ in range(2):
        again = q.linear_backward(G, Xt, Zc, wq, At, Bt, 2.0)
        for a_, b_ in zip(ref, again):
            assert torch.equal(a_, b_)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        on_side = q.linear_backward(G, Xt, Zc, wq, At, Bt, 2.0)
    torch.cuda.current_stream().wait_stream(side)
    for a_, b_ in zip(ref, on_side):
        assert torch.equal(a_, b_)
    # graph capture: outputs, workspace and status allocated before capture
    dX = torch.empty_like(ref[0])
    dA = torch.empty_like(ref[1])
    dB = torch.empty_like(ref[2])
    st = q.new_status()
    ws = torch.empty(int(q.lib.qlora_linear_bwd_workspace_size(M, K, N, r)), dtype=torch.uint8,
                     device="cuda")
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        q.linear_backward(G, Xt, Zc, wq, At, Bt, 2.0, dX=dX, dA=dA, dB=dB, status=st, workspace=ws)
        cap.synchronize()
        with torch.cuda.graph(g, stream=cap):
            q.linear_backward(G, Xt, Zc, wq, At, Bt, 2.0, dX=dX, dA=dA, dB=dB, status=st,
                              workspace=ws)
    torch.cuda.synchronize()
    for t in (dX, dA, dB):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert q.status_sync(st) == (0, 0)
    for a_, b_ in zip(ref, (dX, dA, dB)):
        assert torch.equal(a_, b_)
    del g


GEMV_SHAPES = [
    # (M, K, N, r, dq): K not a multiple of 128 (a half stage of zeros), a ragged
    # last column group, one 64-row stage, no double quantization, a rank wider
    # than the column groups' 8-column slices (X·A by the rank-r kernel), and a
    # single column group with one split per 128 rows
    (1, 576, 576, 16, True),
    (3, 64, 320, 8, False),
    (16, 1088, 1344, 64, True),
    (7, 2112, 256, 8, True),
    (12, 832, 704, 24, False),
]


@pytest.mark.parametrize("M,K,N,r,dq", GEMV_SHAPES)
def test_gemv_shapes(M, K, N, r, dq):
    lin = S.random_case(1000 + M + K + N, M, K, N, r)
    errs = run_case(lin, r, 16.0 / r, dq, backward=False)
    for k, v in errs.items():
        assert v <= TOL, (k, v, errs)


def test_config1_tiny():
    wl = S.config1()
    lin = wl.linears[0]
    errs = run_case(lin, wl.r, wl.c, wl.double_quant, w_dtype=torch.float32)
    for k, v in errs.items():
        assert v <= TOL, (k, v, errs)


def test_special_cases():
    q = _q()
    M, K, N, r = 160, 256, 320, 16
    lin = S.random_case(5, M, K, N, r)
    X, W = lin.X, lin.W
    Xt = to_dev(X)
    wq = q.quantize(to_dev(W), double_quant=True)
    ow = OracleWeight(W, True)
    zA, zB = torch.zeros((K, r), dtype=torch.bfloat16, device="cuda"), \
        torch.zeros((r, N), dtype=torch.bfloat16, device="cuda")
    # A = B = 0: a plain product with the decoded weight
    Y, Zc = q.linear_forward(Xt, wq, zA, zB, 2.0)
    assert rel_fro(to_np(Y), X.astype(np.float64) @ ow.w_hat) <= TOL
    assert torch.count_nonzero(Zc) == 0
    # W = 0: only the LoRA branch remains (every code 7, every weight exactly 0)
    w0 = q.quantize(torch.zeros((K, N), dtype=torch.bfloat16, device="cuda"), double_quant=True)
    At, Bt = to_dev(lin.A), to_dev(lin.B)
    Y, _ = q.linear_forward(Xt, w0, At, Bt, 2.0)
    assert rel_fro(to_np(Y), 2.0 * (X.astype(np.float64) @ lin.A) @ lin.B) <= TOL
    # B = 0: dA is exactly zero while dB is not
    G = S.normal(9, 9, 9, (M, N), 1.0)
    Y, Zc = q.linear_forward(Xt, wq, At, zB, 2.0)
    dX, dA, dB = q.linear_backward(to_dev(G), Xt, Zc, wq, At, zB, 2.0)
    assert torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) > 0


def test_no_gradient_for_the_frozen_base():
    """Backward leaves every buffer of the quantized state untouched."""
    q = _q()
    lin = S.random_case(11, 256, 256, 256, 16)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    before = [t.clone() for t in (wq.packed, wq.code8, wq.s2, wq.offset)]
    Xt = to_dev(lin.X)
    Y, Zc = q.linear_forward(Xt, wq, to_dev(lin.A), to_dev(lin.B), 2.0)
    q.linear_backward(to_dev(lin.dY), Xt, Zc, wq, to_dev(lin.A), to_dev(lin.B), 2.0)
    torch.cuda.synchronize()
    for a, b in zip(before, (wq.packed, wq.code8, wq.s2, wq.offset)):
        assert torch.equal(a, b)


def test_full_size_projection_sampled_rows():
    """4096 x 4096, M = 4096 (the benchmark shape): sampled rows of Y and dX,
    full dA and dB."""
    q = _q()
    wl = S.config2()
    lin = wl.linears[0]
    X, W, A, B, G, c = lin.X, lin.W, lin.A, lin.B, lin.dY, wl.c
    wq = q.quantize(to_dev(W), double_quant=True)
    Xt = to_dev(X)
    Y, Zc = q.linear_forward(Xt, wq, to_dev(A), to_dev(B), c)
    dX, dA, dB = q.linear_backward(to_dev(G), Xt, Zc, wq, to_dev(A), to_dev(B), c)
    ow = OracleWeight(W, True)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 4095], rng.integers(0, 4096, 96)]))
    Yr, _ = lora_forward(X[rows], ow.w_hat, A, B, c)
    assert_close("Y rows", to_np(Y)[rows], Yr)
    dXr, _, _ = lora_backward(G[rows], X[rows], ow.w_hat, A, B, c)
    assert_close("dX rows", to_np(dX)[rows], dXr)
    _, dAr, dBr = lora_adapter_grads(G, X, A, B, c)
    assert_close("dA", to_np(dA), dAr)
    assert_close("dB", to_np(dB), dBr)


# r % 8 == 0 runs the tensor-core tile kernel (128 x 256 tiles; 4160 x 2880
# gives 396 tiles, several per CTA, with a ragged last row and column tile);
# other ranks run the mma.sync kernel
MERGE_CASES = [(64, 128, 8, True), (320, 384, 16, False), (256, 576, 64, True), (128, 64, 24, True),
               (4160, 2880, 32, True), (1088, 1344, 64, False), (192, 320, 12, True), (64, 192, 3, False)]


@pytest.mark.parametrize("K,N,r,dq", MERGE_CASES)
def test_merge_parity(K, N, r, dq):
    """qlora_nf4_merge against the oracle's RN_bf16(W_hat + cAB): every output
    within one bf16 ulp (fp32 rank-r sum on the device), nearly all exact."""
    from oracle.merge import merge_bf16, merge_exact
    q = _q()
    lin = S.random_case(77 + K + N + r, 4, K, N, r)
    c = 16.0 / r
    wq = q.quantize(to_dev(lin.W), double_quant=dq)
    got = to_np(q.merge(wq, to_dev(lin.A), to_dev(lin.B), c))
    ow = OracleWeight(lin.W, dq)
    ref = merge_bf16(ow.w_hat, lin.A, lin.B, c)
    ex = merge_exact(ow.w_hat, lin.A, lin.B, c)
    _, e = np.frexp(np.maximum(np.abs(ex), 1e-30))
    ulp = np.ldexp(1.0, e - 8)
    assert np.all(np.abs(got - ref) <= ulp), float(np.max(np.abs(got - ref) / ulp))
    assert np.mean(got != ref) < 0.01


def test_merge_zero_adapter_is_dequantize():
    q = _q()
    lin = S.random_case(91, 4, 192, 256, 16)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    A = torch.zeros((192, 16), dtype=torch.bfloat16, device="cuda")
    got = q.merge(wq, A, to_dev(lin.B), 2.0)
    assert torch.equal(got, q.dequantize(wq))


def test_merge_requantize_matches_oracle_quantize_of_merged():
    """Re-quantized delivery: the GPU's quantization of its merged weight is the
    oracle's quantization of the same bf16 values, bit for bit."""
    from oracle import nf4
    q = _q()
    lin = S.random_case(93, 4, 128, 256, 16)
    wq = q.quantize(to_dev(lin.W), double_quant=True)
    merged = q.merge(wq, to_dev(lin.A), to_dev(lin.B), 2.0)
    rq = q.merge_requantize(wq, to_dev(lin.A), to_dev(lin.B), 2.0, double_quant=True)
    codes, absmax = nf4.quantize_nf4(to_np(merged).ravel())
    payload, _ = nf4.pack_codes(codes)
    code8, s2, off = nf4.double_quantize(absmax)
    assert np.array_equal(rq.packed.cpu().numpy(), payload)
    assert np.array_equal(rq.code8.cpu().numpy(), code8)

"""Pins of the fp64 linear-layer oracle.

Source: "QLoRA：冻结的 4-bit 权重怎样参与一次微调", §冻结权重为什么仍然需要输入
梯度 and §一次完整反向与有限差分 (worked example, asserts, B = 0 case),
§Merge 后还是不是训练时的函数.  Uniform INT4: "SFT（四）：QLoRA的4-bit量化与
LoRA微调原理" §6.
"""
import numpy as np

from oracle import nf4
from oracle.int4 import int4_quantize_block, int4_dequantize_block
from oracle.linear import lora_backward, lora_forward


def _example(g, B=None):
    w = nf4.dequantize(np.frombuffer(bytes.fromhex(g["packed_hex"]), np.uint8), 2,
                       np.array([g["scale"]], np.float32))
    X = np.array([g["x"]])                    # 1 x 2
    W = w.reshape(2, 1)                       # K=2 x N=1
    A = np.array(g["A"]).reshape(2, 1)        # r = 1
    Bm = np.array([[g["B"] if B is None else B]])
    return X, W, A, Bm


def test_worked_backward_example(golden):
    g = golden("backward_worked_example.json")
    X, W, A, B = _example(g)
    Y, Z = lora_forward(X, W, A, B, g["c"])
    assert abs((X @ W)[0, 0] - g["base_output"]) < 1e-12
    assert abs(g["c"] * (Z @ B)[0, 0] - g["adapter_output"]) < 1e-12
    assert abs(Y[0, 0] - g["y"]) < 1e-12
    G = Y - g["target"]                       # dL/dY of L = (y - target)^2 / 2
    assert abs(G[0, 0] - g["G"]) < 1e-12
    dX, dA, dB = lora_backward(G, X, W, A, B, g["c"])
    assert np.allclose(dX.ravel(), g["dX"], rtol=0, atol=1e-12)
    assert np.allclose(dA.ravel(), g["dA"], rtol=0, atol=1e-12)
    assert abs(dB[0, 0] - g["dB"]) < 1e-12
    # B = 0: dA vanishes exactly, dB does not
    X, W, A, B0 = _example(g, B=0.0)
    Y0, _ = lora_forward(X, W, A, B0, g["c"])
    dX0, dA0, dB0 = lora_backward(Y0 - g["target"], X, W, A, B0, g["c"])
    assert np.all(dA0 == 0.0) and list(dA0.ravel()) == g["B_zero_dA"]
    assert dB0[0, 0] != 0.0


def test_worked_example_central_differences(golden):
    g = golden("backward_worked_example.json")
    X, W, A, B = _example(g)
    c, t, eps = g["c"], g["target"], g["fd_eps"]

    def loss(p):
        Y, _ = lora_forward(p[:2].reshape(1, 2), W, p[2:4].reshape(2, 1), p[4:].reshape(1, 1), c)
        return 0.5 * (Y[0, 0] - t) ** 2

    p0 = np.concatenate([X.ravel(), A.ravel(), B.ravel()])
    Y, _ = lora_forward(X, W, A, B, c)
    dX, dA, dB = lora_backward(Y - t, X, W, A, B, c)
    analytic = np.concatenate([dX.ravel(), dA.ravel(), dB.ravel()])
    for i, want in enumerate(analytic):
        pp, pm = p0.copy(), p0.copy()
        pp[i] += eps
        pm[i] -= eps
        num = (loss(pp) - loss(pm)) / (2 * eps)
        assert abs(num - want) <= max(g["fd_rel_tol"] * max(abs(num), abs(want)), g["fd_abs_tol"])


def test_random_shapes_central_differences():
    rng = np.random.default_rng(11)
    for (M, K, N, r) in [(3, 5, 4, 2), (1, 7, 3, 1), (4, 4, 6, 3)]:
        X, W = rng.standard_normal((M, K)), rng.standard_normal((K, N))
        A, B = rng.standard_normal((K, r)), rng.standard_normal((r, N))
        R = rng.standard_normal((M, N))
        c = 0.75

        def L(X_, A_, B_):
            return float(np.sum(lora_forward(X_, W, A_, B_, c)[0] * R))

        dX, dA, dB = lora_backward(R, X, W, A, B, c)
        for arr, grad, which in ((X, dX, 0), (A, dA, 1), (B, dB, 2)):
            for idx in np.ndindex(arr.shape):
                h = 1e-6
                args_p = [X.copy(), A.copy(), B.copy()]
                args_m = [X.copy(), A.copy(), B.copy()]
                args_p[which][idx] += h
                args_m[which][idx] -= h
                num = (L(*args_p) - L(*args_m)) / (2 * h)
                assert abs(num - grad[idx]) <= 1e-6 * max(1.0, abs(num))


def test_special_cases_reduce_to_plain_products():
    rng = np.random.default_rng(12)
    M, K, N, r = 3, 4, 5, 2
    X, W = rng.standard_normal((M, K)), rng.standard_normal((K, N))
    Z0A, Z0B = np.zeros((K, r)), np.zeros((r, N))
    Y, _ = lora_forward(X, W, Z0A, Z0B, 2.0)
    want = np.array([[sum(X[m, k] * W[k, n] for k in range(K)) for n in range(N)] for m in range(M)])
    assert np.allclose(Y, want, rtol=1e-14, atol=1e-14)
    A, B = rng.standard_normal((K, r)), rng.standard_normal((r, N))
    Y, Z = lora_forward(X, np.zeros((K, N)), A, B, 2.0)
    want = 2.0 * np.array([[sum(sum(X[m, k] * A[k, j] for k in range(K)) * B[j, n]
                                for j in range(r)) for n in range(N)] for m in range(M)])
    assert np.allclose(Y, want, rtol=1e-13, atol=1e-13)
    # merged weight: X (W + c A B) equals the two-branch output
    Y2, _ = lora_forward(X, W, A, B, 0.5)
    assert np.allclose(Y2, X @ (W + 0.5 * A @ B), rtol=1e-13, atol=1e-13)
    # dX with A = B = 0 is G W^T; dA is then 0
    G = rng.standard_normal((M, N))
    dX, dA, dB = lora_backward(G, X, W, Z0A, Z0B, 1.0)
    assert np.allclose(dX, np.array([[sum(G[m, n] * W[k, n] for n in range(N)) for k in range(K)]
                                     for m in range(M)]), rtol=1e-14, atol=1e-14)
    assert np.all(dA == 0) and np.all(dB == 0)


def test_int4_uniform_worked_example(golden):
    g = golden("int4_uniform_example.json")
    q, s = int4_quantize_block(g["W"])
    assert q == g["q"]
    assert abs(s - g["s_approx"]) < 1e-4
    w_hat = int4_dequantize_block(q, s)
    tol = g["approx_abs_tol"]
    assert all(abs(a - b) < tol for a, b in zip(w_hat, g["w_hat_approx"]))
    assert all(abs((w - h) - e) < tol for w, h, e in zip(g["W"], w_hat, g["error_approx"]))


def test_int4_library_format_worked_example(golden):
    """The stored format reproduces the page's example: q = [-7, -2, 1, 5]
    (codes q + 8), scale ~0.1714, reconstruction ~[-1.200, -0.343, 0.171, 0.857]."""
    from oracle.int4 import int4_dequantize, int4_quantize
    g = golden("int4_uniform_example.json")
    codes, s = int4_quantize(np.array(g["W"], dtype=np.float32))
    assert list(codes.astype(int) - 8) == g["q"]
    assert abs(float(s[0]) - g["s_approx"]) < 1e-4
    w_hat = int4_dequantize(codes, s)
    # the reconstruction is rounded to bf16 (3 significant digits)
    assert np.all(np.abs(w_hat - np.array(g["w_hat_approx"])) < 5e-3)


def test_int4_library_format_against_block_rule():
    """Same codes as the fp64 per-block rule except where w/s sits within the
    fp32 rounding of s from a .5 tie; all-zero blocks get scale 1; padding 8."""
    from oracle.int4 import int4_quantize
    rng = np.random.default_rng(8)
    w = rng.normal(0, 0.02, 64 * 500).astype(np.float32)
    w[64 * 7:64 * 8] = 0.0
    codes, s = int4_quantize(w)
    assert s[7] == 1.0 and np.all(codes[64 * 7:64 * 8] == 8)
    agree = 0
    for b in range(500):
        q_ref, s_ref = int4_quantize_block(w[64 * b:64 * b + 64])
        q = list(codes[64 * b:64 * b + 64].astype(int) - 8)
        agree += sum(int(a == c) for a, c in zip(q, q_ref))
        assert abs(float(s[b]) - s_ref) <= 2 ** -23 * s_ref
    assert agree >= 64 * 500 - 5
    # brute force on a tiny block: every q is the nearest integer (ties away
    # from zero) of w / s within [-7, 7]
    w = np.array([0.7, -0.05, 0.35, 0.0, -0.7, 0.2499], dtype=np.float32)
    codes, s = int4_quantize(w)
    for v, c in zip(w.astype(np.float64), codes.astype(int)):
        t = v / float(s[0])
        cands = list(range(-7, 8))
        best = min(cands, key=lambda q: (abs(t - q), -abs(q)))
        assert c - 8 == best


def test_int4_ties_round_half_away_from_zero():
    """The page does not say how round() breaks a tie; the reading taken is
    half away from zero (the school rule).  With amax = 7 the scale is 1 and
    w / s are exact halves."""
    from oracle.int4 import int4_quantize
    vals = [7.0, 2.5, -2.5, 0.5, -0.5, 1.5, -6.5]
    want = [7, 3, -3, 1, -1, 2, -7]
    q, s = int4_quantize_block(vals)
    assert s == 1.0 and q == want
    codes, sc = int4_quantize(np.array(vals, dtype=np.float32))
    assert float(sc[0]) == 1.0 and list(codes.astype(int) - 8) == want


def test_int4_dequantize_is_one_bf16_rounding_of_q_times_s():
    """Decoded weights are bf16 values within half a bf16 ulp of the exact
    q * s (s = RN_fp32(amax / 7) is not a bf16 number in general)."""
    from oracle.int4 import int4_dequantize, int4_quantize
    rng = np.random.default_rng(12)
    w = rng.normal(0, 0.02, 64 * 50).astype(np.float32)
    codes, s = int4_quantize(w)
    out = int4_dequantize(codes, s)
    exact = (codes.astype(np.float64) - 8) * s.astype(np.float64)[np.arange(w.size) // 64]
    f32 = out.astype(np.float32)
    assert np.all(f32.astype(np.float64) == out)               # fp32-exact
    assert np.all((f32.view(np.uint32) & 0xFFFF) == 0)          # and bf16-exact
    nz = exact != 0
    _, e = np.frexp(exact[nz])
    half_ulp = np.ldexp(1.0, e - 9)                             # bf16: 8 significant bits
    assert np.all(np.abs(out[nz] - exact[nz]) <= half_ulp)
    assert np.any(out[nz] != exact[nz])                         # rounding does happen
    assert np.all(out[~nz] == 0)


def test_int4_ragged_tail_block():
    """The stored format's last block holds only the tail: its scale comes
    from the tail alone, and an all-zero tail gets scale 1 and code 8 (q = 0)."""
    from oracle.int4 import int4_quantize
    w = np.full(64 + 3, 0.01, np.float32)
    w[63] = 5.0
    w[64:] = [0.7, -0.3, 0.12]                  # no w / s near a .5 tie
    codes, s = int4_quantize(w)
    q_ref, s_ref = int4_quantize_block(w[64:])
    assert abs(float(s[1]) - s_ref) <= 2 ** -23 * s_ref
    assert list(codes[64:].astype(int) - 8) == q_ref == [7, -3, 1]
    w[64:] = 0.0
    codes, s = int4_quantize(w)
    assert float(s[1]) == 1.0 and np.all(codes[64:] == 8)


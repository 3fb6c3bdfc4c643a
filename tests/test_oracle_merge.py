"""Pins of the merge/export oracle (``oracle/merge.py``)."""
import numpy as np

from oracle import nf4
from oracle.linear import lora_forward
from oracle.merge import merge_bf16, merge_exact


def test_page_merge_example(golden):
    g = golden("merge_requant_example.json")
    W_hat = np.array(g["w_hat"], dtype=np.float64).reshape(2, 1)    # K = 2, N = 1
    A = np.array(g["A"], dtype=np.float64).reshape(2, 1)            # r = 1
    B = np.array([[g["B"]]], dtype=np.float64)
    merged = merge_exact(W_hat, A, B, g["c"])
    assert np.allclose(merged.ravel() - W_hat.ravel(), g["cAB"], rtol=0, atol=1e-15)
    assert np.allclose(merged.ravel(), g["merged"], rtol=0, atol=1e-15)
    x = np.array(g["x"], dtype=np.float64)
    assert abs(float(x @ merged.ravel()) - g["merged_output"]) < 1e-15
    # the merged function equals the trained one (the adapter's output added)
    y, _ = lora_forward(x.reshape(1, 2), W_hat, A, B, g["c"])
    assert abs(float(y[0, 0]) - g["merged_output"]) < 1e-15


def test_merged_function_equals_training_function():
    rng = np.random.default_rng(3)
    for (M, K, N, r) in ((5, 64, 128, 8), (3, 192, 64, 16), (7, 128, 192, 64)):
        W = nf4.round_to_bf16(rng.normal(0, 0.02, (K, N)))
        A = nf4.round_to_bf16(rng.normal(0, 0.01, (K, r)))
        B = nf4.round_to_bf16(rng.normal(0, 0.01, (r, N)))
        X = nf4.round_to_bf16(rng.normal(0, 1, (M, K)))
        c = 32.0 / r
        y, _ = lora_forward(X, W, A, B, c)
        y2 = X @ merge_exact(W, A, B, c)
        assert np.max(np.abs(y - y2)) <= 1e-12 * max(1.0, np.max(np.abs(y)))


def test_zero_adapter_and_rounding():
    rng = np.random.default_rng(4)
    W = nf4.round_to_bf16(rng.normal(0, 0.02, (64, 128)))
    A = np.zeros((64, 16))
    B = nf4.round_to_bf16(rng.normal(0, 0.01, (16, 128)))
    assert np.array_equal(merge_bf16(W, A, B, 2.0), W)
    # delivered values are bf16 and within half a bf16 ulp of the exact merge
    A = nf4.round_to_bf16(rng.normal(0, 0.01, (64, 16)))
    ex = merge_exact(W, A, B, 2.0)
    m = merge_bf16(W, A, B, 2.0)
    assert np.array_equal(nf4.round_to_bf16(m), m)
    _, e = np.frexp(ex)
    half_ulp = np.ldexp(1.0, e - 9)
    assert np.all(np.abs(m - ex) <= half_ulp)

"""Pins for the oracle's projections (step 2 and the GEMV of steps 9+10+11 of the
page "spark_model/forward/qwen3_5/linear_attention.rs"): a hand-worked product,
one-hot weights that select input columns, linearity, and the routing of the stacked
in_proj weight rows (qkv | z | a | b) to the four outputs."""
import numpy as np

import oracle
from gated_delta_rule_102_b200 import synth

bf = synth.to_bf16_bits


def test_hand_worked_2x3():
    # x = [[1, 2, 3], [-1, 0.5, 2]], W = [[1, 0, -1], [2, 1, 0.5]] (rows = outputs):
    # out[0] = (1 - 3, 2 + 2 + 1.5) = (-2, 5.5); out[1] = (-1 - 2, -2 + 0.5 + 1) = (-3, -0.5)
    x = bf(np.array([[1, 2, 3], [-1, 0.5, 2]]))
    w = bf(np.array([[1, 0, -1], [2, 1, 0.5]]))
    np.testing.assert_array_equal(oracle.linear(x, w), [[-2.0, 5.5], [-3.0, -0.5]])


def test_one_hot_rows_select_input_columns_exactly():
    rng = np.random.default_rng(31)
    R, K, N = 5, 24, 7
    x = bf(rng.normal(size=(R, K)))
    pick = rng.integers(0, K, N)
    w = np.zeros((N, K))
    w[np.arange(N), pick] = 1.0
    np.testing.assert_array_equal(oracle.linear(x, bf(w)), oracle.bf16_to_f64(x)[:, pick])


def test_linear_in_the_input_and_transposition_sensitive():
    rng = np.random.default_rng(32)
    R, K, N = 3, 16, 5
    x1, x2 = rng.integers(-8, 8, (R, K)).astype(float), rng.integers(-8, 8, (R, K)).astype(float)
    w = bf(rng.normal(size=(N, K)))
    y = oracle.linear(bf(x1 + x2), w)
    np.testing.assert_allclose(y, oracle.linear(bf(x1), w) + oracle.linear(bf(x2), w), rtol=0, atol=1e-12)
    assert y.shape == (R, N)


def test_in_proj_routes_the_stacked_weight_rows():
    sh = oracle.Shape(2, 4, 16, 8, 4)           # C = 2*2*16 + 4*8 = 96, Z = 32, Hv = 4
    C, Z, Hv, hidden = 96, 32, 4, 40
    N = C + Z + 2 * Hv
    rng = np.random.default_rng(33)
    x = bf(rng.normal(size=(3, hidden)))
    w = np.zeros((N, hidden))
    w[np.arange(N), np.arange(N) % hidden] = 1.0  # output feature n reads input column n % hidden
    r = oracle.in_proj(sh, x, bf(w))
    xv = oracle.bf16_to_f64(x)
    col = lambda lo, n: xv[:, np.arange(lo, lo + n) % hidden]  # noqa: E731
    np.testing.assert_array_equal(r["qkv"], col(0, C))
    np.testing.assert_array_equal(r["z"], col(C, Z))
    np.testing.assert_array_equal(r["a"], col(C + Z, Hv))
    np.testing.assert_array_equal(r["b"], col(C + Z + Hv, Hv))


def test_out_proj_shape_and_value():
    sh = oracle.Shape(1, 2, 16, 8, 4)            # Hv*dv = 16
    rng = np.random.default_rng(34)
    y = bf(rng.normal(size=(2, 16)))
    w = bf(rng.normal(size=(6, 16)))
    out = oracle.out_proj(sh, y, w)
    ref = np.array([[sum(oracle.bf16_to_f64(y)[r, k] * oracle.bf16_to_f64(w)[n, k] for k in range(16))
                     for n in range(6)] for r in range(2)])  # the sum written as a loop, for two rows
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)

"""The chunked form of the multi-token step, restated in numpy and checked against the
oracle's token-by-token delta rule (step 7 of the page
"spark_model/forward/qwen3_5/linear_attention.rs", applied token after token).

For one (sequence, head) with S0 the state before the launch and n tokens:
  gamma_t = alpha_0 ... alpha_t,  g_ts = alpha_{s+1} ... alpha_t,  w_s = g_{n-1,s}
  delta_t = beta_t (v_t - gamma_t S0^T k_t) - sum_{s<t} beta_t g_ts (k_s.k_t) delta_s
  o_t     = gamma_t S0^T q_t + sum_{s<=t} g_ts (q_t.k_s) delta_s
  S_n     = gamma_{n-1} S0 + sum_s w_s k_s delta_s^T
This is what the tensor-core multi-token kernel computes (two contractions and a 16 x 16
triangular solve). In exact arithmetic it equals the recurrence, so in fp64 it must match
the oracle to rounding; with the two contractions done as the tensor core does them
(operands truncated to tf32, each split into a high part and the remainder, three
products) it must stay far inside the parity bars, while one tf32 product alone would
not."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def tf32(x):
    """fp32 bit pattern read as tf32: the low 13 mantissa bits dropped (truncation)."""
    b = np.asarray(x, np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return b.view(np.float32).astype(np.float64)


def split(x):
    x32 = np.asarray(x, np.float32)
    hi = tf32(x32)
    lo = (x32.astype(np.float64) - hi).astype(np.float32)  # exact in fp32
    return hi, tf32(lo)


def matmul(a, b, mode):
    if mode == "exact":
        return a @ b
    ah, al = split(a)
    bh, bl = split(b)
    if mode == "tf32x3":
        return ah @ bh + ah @ bl + al @ bh
    return ah @ bh  # "tf32x1"


def chunk_form(q, k, v, alpha, beta, S0, n, mode="exact"):
    """q, k [T][dk], v [T][dv], alpha, beta [T], S0 [dk][dv]; tokens >= n are ignored."""
    T, dv = v.shape
    idx = np.arange(T)
    a = np.where(idx < n, alpha, 1.0)
    b = np.where(idx < n, beta, 0.0)
    gamma = np.array([np.prod(a[:t + 1]) for t in range(T)])
    g = np.zeros((T, T))
    for t in range(T):
        for s in range(t + 1):
            g[t, s] = np.prod(a[s + 1:t + 1])
    KK, QK = k @ k.T, q @ k.T
    UP = matmul(np.concatenate([k, q]), S0, mode)  # rows: S0^T k_t, then S0^T q_t
    U, P = UP[:T], UP[T:]
    delta, o = np.zeros((T, dv)), np.zeros((T, dv))
    for t in range(n):
        x = b[t] * (v[t] - gamma[t] * U[t])
        for s in range(t):
            x -= b[t] * g[t, s] * KK[t, s] * delta[s]
        delta[t] = x
        y = gamma[t] * P[t]
        for s in range(t + 1):
            y += g[t, s] * QK[t, s] * delta[s]
        o[t] = y
    w = np.array([np.prod(a[s + 1:n]) if s < n else 0.0 for s in range(T)])
    S = gamma[n - 1] * S0 + matmul(k.T, w[:, None] * delta, mode)
    return o[:n], S, delta[:n]


def problem(rng, T, dk, dv, decay="normal", s_std=0.02):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True) * np.sqrt(dk)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv)) * 0.5
    if decay == "normal":
        alpha = np.exp(-rng.uniform(0.0, 0.5, T))
    else:  # from 1 down to far below fp32's range
        alpha = 2.0 ** -rng.choice([0.0, 1.0, 10.0, 48.0, 200.0], T)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    S0 = rng.standard_normal((dk, dv)) * s_std
    return q, k, v, alpha, beta, S0


def oracle_tokens(q, k, v, alpha, beta, S0, n):
    dk, dv = S0.shape
    sh = oracle.Shape(1, 1, dk, dv, 4)
    pool = S0[None, None].copy()
    o = oracle.delta_rule(sh, q[None, :n, None], k[None, :n, None], v[None, :n, None], alpha[None, :n, None],
                          beta[None, :n, None], pool, np.zeros(1, np.int32))
    return o[0, :, 0], pool[0, 0]


@pytest.mark.parametrize("T,n,decay", [(16, 16, "normal"), (16, 5, "normal"), (16, 1, "normal"),
                                       (7, 7, "wide"), (16, 16, "wide")])
def test_chunk_form_equals_the_recurrence_in_fp64(T, n, decay):
    rng = np.random.default_rng(1000 * T + 10 * n + (decay == "wide"))
    q, k, v, alpha, beta, S0 = problem(rng, T, 32, 48, decay)
    o, S, _ = chunk_form(q, k, v, alpha, beta, S0, n)
    o_ref, S_ref = oracle_tokens(q, k, v, alpha, beta, S0, n)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12 * max(1.0, np.abs(o_ref).max()))
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-12 * max(1.0, np.abs(S_ref).max()))


def test_tokens_past_n_change_nothing():
    # the kernel pads every sequence to 16 tokens: decays 1, strengths 0 past its count
    rng = np.random.default_rng(7)
    q, k, v, alpha, beta, S0 = problem(rng, 16, 16, 16)
    o5, S5, d5 = chunk_form(q, k, v, alpha, beta, S0, 5)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[5:], k2[5:], v2[5:] = 3.0, -2.0, 7.0  # garbage past the count
    o5b, S5b, d5b = chunk_form(q2, k2, v2, alpha, beta, S0, 5)
    np.testing.assert_array_equal(o5, o5b)
    np.testing.assert_array_equal(S5, S5b)


@pytest.mark.parametrize("s_std", [0.02, 1.0])
def test_split_tf32_products_stay_inside_the_bars(s_std):
    # dk = dv = 128, 16 tokens: the kernel's shape. Bars: state within 1e-4 of the head's
    # largest entry; outputs (before the RMSNorm, relative to their largest) well under it.
    rng = np.random.default_rng(11 + int(s_std))
    q, k, v, alpha, beta, S0 = problem(rng, 16, 128, 128, s_std=s_std)
    o_ref, S_ref = oracle_tokens(q, k, v, alpha, beta, S0, 16)
    o3, S3, _ = chunk_form(q, k, v, alpha, beta, S0, 16, mode="tf32x3")
    o1, S1, _ = chunk_form(q, k, v, alpha, beta, S0, 16, mode="tf32x1")
    err3 = np.abs(S3 - S_ref).max() / np.abs(S_ref).max()
    err1 = np.abs(S1 - S_ref).max() / np.abs(S_ref).max()
    oerr3 = np.abs(o3 - o_ref).max() / np.abs(o_ref).max()
    assert err3 < 2e-6 and oerr3 < 2e-6, (err3, oerr3)
    assert err1 > 10 * err3  # one truncated product is not enough


def test_chunk_form_equals_the_recurrence_on_random_shapes():
    # token counts 1..16 with every partial count, head sizes 8..64, decays from near 1 down to
    # far below fp32's range, strengths 0..1, state scales 0..1
    rng = np.random.default_rng(2024)
    for case in range(40):
        T = int(rng.integers(1, 17))
        n = int(rng.integers(1, T + 1))
        dk, dv = (int(x) for x in rng.choice([8, 16, 32, 64], 2))
        decay = "wide" if case % 3 == 0 else "normal"
        q, k, v, alpha, beta, S0 = problem(rng, T, dk, dv, decay, s_std=float(rng.choice([0.0, 0.02, 1.0])))
        if case % 5 == 0:
            beta[rng.integers(0, T)] = 0.0  # a token that writes nothing
        o, S, _ = chunk_form(q, k, v, alpha, beta, S0, n)
        o_ref, S_ref = oracle_tokens(q, k, v, alpha, beta, S0, n)
        scale_o, scale_s = max(1.0, np.abs(o_ref).max()), max(1.0, np.abs(S_ref).max())
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12 * scale_o, err_msg=f"case {case}: T={T} n={n}")
        np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-12 * scale_s, err_msg=f"case {case}: T={T} n={n}")

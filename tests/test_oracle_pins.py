"""Pins for the FP64 oracle: checks against facts the method and the mathematics
fix, independent of the oracle's own code (closed forms, identities, hand-worked
examples, invariants, structural permutations).

Method source: the page "spark_model/forward/qwen3_5/linear_attention.rs",
steps 3 (fused causal conv1d update + L2 norm), 4 (gate), 5 (beta), 6 (Q|K|V
split), 7 (gated_delta_rule_decode), 8 (per-head RMSNorm) and the SiLU(z) gate
of steps 9+10+11.
"""
import math

import numpy as np
import pytest

import oracle
from gated_delta_rule_102_b200 import synth

bf = synth.to_bf16_bits
unbf = lambda h: synth.bf16_bits_to_f32(h).astype(np.float64)  # noqa: E731


def _shape(Hk=1, Hv=1, dk=2, dv=2, W=4, **kw):
    return oracle.Shape(Hk, Hv, dk, dv, W, **kw)


# --------------------------------------------------------------------------- step 7
def _run_delta(S0, steps, matrix_form=False):
    """Run the oracle's delta rule for one head (Hk = Hv = 1), T=1 per call."""
    dk, dv = S0.shape
    sh = _shape(dk=dk, dv=dv)
    pool = np.ascontiguousarray(S0, dtype=np.float64).reshape(1, 1, dk, dv).copy()
    outs = []
    fn = oracle.delta_rule_matrix_form if matrix_form else oracle.delta_rule
    for st in steps:
        q = np.array(st["q"], float).reshape(1, 1, 1, dk)
        k = np.array(st["k"], float).reshape(1, 1, 1, dk)
        v = np.array(st["v"], float).reshape(1, 1, 1, dv)
        al = np.array([[[st["alpha"]]]])
        be = np.array([[[st["beta"]]]])
        outs.append(fn(sh, q, k, v, al, be, pool, [0])[0, 0, 0])
    return pool[0, 0], outs


# The three steps below were worked out by hand, one scalar at a time, from
# S <- alpha S; m = S^T k; delta = beta (v - m); S <- S + k delta^T; o = S^T q
# with S indexed [key dim i][value dim j]:
#  step 1: alpha S = [[.5,1],[1.5,2]]; m = row0 = (.5,1); delta = .5*(1.5,3) = (.75,1.5);
#          row0 += delta -> [[1.25,2.5],[1.5,2]]; o = row1 = (1.5,2)
#  step 2: m = row1 = (1.5,2); delta = (-2.5,-1.5); row1 += delta -> [[1.25,2.5],[-1,.5]];
#          o = row0 + row1 = (.25,3)
#  step 3: alpha S = [[.3125,.625],[-.25,.125]]; m = .6 row0 + .8 row1 = (-.0125,.475);
#          delta = .5*(1.0125,-2.475) = (.50625,-1.2375);
#          S = [[.3125+.30375, .625-.7425],[-.25+.405, .125-.99]] = [[.61625,-.1175],[.155,-.865]];
#          o = .8 row0 - .6 row1 = (.493-.093, -.094+.519) = (.4,.425)
HAND_STEPS = [
    dict(alpha=0.5, beta=0.5, k=(1, 0), v=(2, 4), q=(0, 1)),
    dict(alpha=1.0, beta=1.0, k=(0, 1), v=(-1, 0.5), q=(1, 1)),
    dict(alpha=0.25, beta=0.5, k=(0.6, 0.8), v=(1, -2), q=(0.8, -0.6)),
]
HAND_O = [(1.5, 2.0), (0.25, 3.0), (0.4, 0.425)]
HAND_S = [[0.61625, -0.1175], [0.155, -0.865]]


@pytest.mark.parametrize("matrix_form", [False, True])
def test_delta_rule_hand_worked_d2(matrix_form):
    S, outs = _run_delta(np.array([[1.0, 2.0], [3.0, 4.0]]), HAND_STEPS, matrix_form)
    for o, want in zip(outs, HAND_O):
        np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, HAND_S, rtol=0, atol=1e-12)


@pytest.mark.parametrize("matrix_form", [False, True])
def test_delta_rule_hand_worked_rectangular(matrix_form):
    # dk=2, dv=3 by hand: alpha S = [[.5,0,-.5],[1,.5,0]]; m = row1 = (1,.5,0);
    # delta = 1*((1,1,1) - m) = (0,.5,1); row1 += delta -> [[.5,0,-.5],[1,1,1]]; o = row0.
    S, outs = _run_delta(np.array([[1.0, 0.0, -1.0], [2.0, 1.0, 0.0]]),
                         [dict(alpha=0.5, beta=1.0, k=(0, 1), v=(1, 1, 1), q=(1, 0))], matrix_form)
    np.testing.assert_array_equal(S, [[0.5, 0.0, -0.5], [1.0, 1.0, 1.0]])
    np.testing.assert_array_equal(outs[0], [0.5, 0.0, -0.5])


def test_no_decay_no_write_leaves_state_bit_identical():
    rng = np.random.default_rng(1)
    S0 = rng.standard_normal((5, 3))
    q, k, v = rng.standard_normal(5), rng.standard_normal(5), rng.standard_normal(3)
    S, outs = _run_delta(S0, [dict(alpha=1.0, beta=0.0, k=k, v=v, q=q)])
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(outs[0], S0.T @ q, rtol=1e-14, atol=1e-14)


def test_beta_zero_is_pure_decay():
    rng = np.random.default_rng(2)
    S0 = rng.standard_normal((4, 6))
    S, _ = _run_delta(S0, [dict(alpha=0.37, beta=0.0, k=rng.standard_normal(4),
                                v=rng.standard_normal(6), q=rng.standard_normal(4))])
    np.testing.assert_array_equal(S, S0 * 0.37)


def test_unit_key_full_write_recalls_value():
    # g = 0, beta = 1, |k| = 1  =>  S'^T k = S^T k + (v - S^T k) k^T k = v.
    rng = np.random.default_rng(3)
    for dk, dv in [(5, 3), (16, 16), (7, 11)]:
        S0 = rng.standard_normal((dk, dv))
        k = rng.standard_normal(dk)
        k /= np.linalg.norm(k)
        v = rng.standard_normal(dv)
        S, _ = _run_delta(S0, [dict(alpha=1.0, beta=1.0, k=k, v=v, q=rng.standard_normal(dk))])
        np.testing.assert_allclose(S.T @ k, v, rtol=0, atol=1e-12)
        # directions orthogonal to k are untouched: S' x = S x for x ⟂ k
        x = rng.standard_normal(dk)
        x -= (x @ k) * k
        np.testing.assert_allclose(S.T @ x, S0.T @ x, rtol=0, atol=1e-12)


def test_contraction_bound():
    # eigenvalues of I - beta k k^T lie in [1 - beta, 1] for |k| = 1, so
    # ||S'||_2 <= alpha ||S||_2 + beta ||k|| ||v||.
    rng = np.random.default_rng(4)
    for _ in range(20):
        S0 = rng.standard_normal((8, 6))
        k = rng.standard_normal(8)
        k /= np.linalg.norm(k)
        v = rng.standard_normal(6)
        al, be = rng.uniform(0.05, 1.0), rng.uniform(0.0, 1.0)
        S, _ = _run_delta(S0, [dict(alpha=al, beta=be, k=k, v=v, q=k)])
        assert np.linalg.norm(S, 2) <= al * np.linalg.norm(S0, 2) + be * np.linalg.norm(v) + 1e-12


def test_two_forms_of_the_update_agree():
    rng = np.random.default_rng(5)
    sh = _shape(Hk=2, Hv=4, dk=6, dv=5)
    B, T, P = 3, 4, 5
    slots = np.array([4, 0, 2], np.int32)
    q = rng.standard_normal((B, T, 2, 6))
    k = rng.standard_normal((B, T, 2, 6))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, 4, 5))
    al = rng.uniform(0.3, 1.0, (B, T, 4))
    be = rng.uniform(0.0, 1.0, (B, T, 4))
    pool = rng.standard_normal((P, 4, 6, 5))
    p1, p2 = pool.copy(), pool.copy()
    o1 = oracle.delta_rule(sh, q, k, v, al, be, p1, slots)
    o2 = oracle.delta_rule_matrix_form(sh, q, k, v, al, be, p2, slots)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(p1, p2, rtol=0, atol=1e-12)
    # slot 1 and slot 3 belong to no sequence: untouched
    np.testing.assert_array_equal(p1[[1, 3]], pool[[1, 3]])


# --------------------------------------------------------------------------- steps 4, 5
def test_gate_closed_forms():
    sh = _shape(Hk=1, Hv=6)
    a_vals = np.array([-4.0, -1.0, 0.0, 0.5, 2.0, 8.0])
    A_log = np.array([0.0, 0.0, 0.0, 0.5, -0.7, 1.0], np.float32)
    dt_bias = np.array([0.0, 0.25, 0.0, -0.125, 0.1, -0.3], np.float32)
    b_vals = np.array([0.0, 1.0, -1.0, 3.0, -2.5, 0.5])
    al, be = oracle.gate(sh, bf(a_vals).reshape(1, 6), bf(b_vals).reshape(1, 6), A_log, dt_bias)
    x = a_vals + dt_bias.astype(np.float64)
    # exp(-softplus(x)) = 1 / (1 + e^x), hence alpha = (1 + e^x)^(-exp(A_log))
    want_alpha = (1.0 + np.exp(x)) ** (-np.exp(A_log.astype(np.float64)))
    np.testing.assert_allclose(al[0], want_alpha, rtol=1e-13)
    assert al[0, 2] == pytest.approx(0.5, abs=1e-15)  # A_log=0, a+dt=0: g = -ln 2
    # beta = sigmoid(b): logit identity beta / (1 - beta) = e^b
    np.testing.assert_allclose(be[0] / (1.0 - be[0]), np.exp(b_vals), rtol=1e-13)
    assert be[0, 0] == 0.5
    # decay in (0, 1) and decreasing in a
    assert np.all((al > 0) & (al < 1))


def test_gate_extremes():
    sh = _shape(Hk=1, Hv=2)
    a = bf(np.array([[60.0, -60.0]]))
    al, _ = oracle.gate(sh, a, bf(np.zeros((1, 2))), np.zeros(2, np.float32), np.zeros(2, np.float32))
    # softplus(60) = 60 (to 1e-26), softplus(-60) = e^-60: no overflow, no lost tail
    assert al[0, 0] == pytest.approx(math.exp(-60.0), rel=1e-14)
    assert al[0, 1] == pytest.approx(math.exp(-math.exp(-60.0)), rel=1e-15)
    # A_log = -inf: the decay is exactly 1; b = -inf: beta is exactly 0
    al, be = oracle.gate(sh, bf(np.array([[1.0, -3.0]])), bf(np.array([[-np.inf, -np.inf]])),
                         np.full(2, -np.inf, np.float32), np.zeros(2, np.float32))
    assert np.all(al == 1.0) and np.all(be == 0.0)


# --------------------------------------------------------------------------- step 3
def _conv_run(sh, x_steps, w, hist0):
    """Feed x_steps (list of [T][C] float arrays) through the oracle's conv for one
    sequence, returning q, k, v per call and the final history."""
    C = sh.channels
    pool = bf(hist0).reshape(1, sh.conv_width - 1, C).copy()
    res = []
    for x in x_steps:
        x = np.asarray(x, float).reshape(1, -1, C)
        res.append(oracle.conv_update(sh, bf(x), bf(w), pool, [0]))
    return res, pool


def test_silu_identities_through_v_channels():
    # one-hot weight on the current tap: v = silu(x). silu(x) - silu(-x) = x,
    # silu(0) = 0, silu(x)/x -> 1 for large x, and silu(x) -> 0 for very negative x.
    sh = _shape(Hk=1, Hv=1, dk=16, dv=16, W=4)
    C = sh.channels
    w = np.zeros((C, 4))
    w[:, 3] = 1.0
    xs = np.array([0.0, 0.5, -0.5, 1.0, -1.0, 2.0, -2.0, 3.0, -3.0, 30.0, -30.0, 0.25, -0.25, 4.0, -4.0, 1.5])
    x = np.zeros(C)
    x[32:48] = xs
    (r,), _ = _conv_run(sh, [x[None]], w, np.zeros((3, C)))
    v = r[2][0, 0, 0]
    assert v[0] == 0.0
    for i in range(1, 15, 2):
        assert v[i] - v[i + 1] == pytest.approx(xs[i], rel=4e-16, abs=1e-15)
    assert v[9] == pytest.approx(30.0, rel=1e-12) and abs(v[10]) < 1e-11


def test_conv_taps_shift_and_history_roll():
    # one-hot weight at tap j reproduces the input W-1-j tokens earlier; the
    # history after the call is the last W-1 raw inputs, bit for bit.
    sh = _shape(Hk=1, Hv=1, dk=16, dv=16, W=4)
    C = sh.channels
    rng = np.random.default_rng(6)
    hist0 = rng.standard_normal((3, C))
    xs = [rng.standard_normal((1, C)) for _ in range(3)] + [rng.standard_normal((2, C))]
    w_cur = np.zeros((C, 4))
    w_cur[:, 3] = 1.0
    ref, _ = _conv_run(sh, xs, w_cur, hist0)
    ref_v = np.concatenate([r[2][0] for r in ref])          # [5 tokens][1][16]: f(x_t)
    raw = np.concatenate([bf(hist0)] + [bf(x) for x in xs])  # 3 history rows then 5 tokens
    for j in range(4):
        w = np.zeros((C, 4))
        w[:, j] = 1.0
        out, pool = _conv_run(sh, xs, w, hist0)
        got_v = np.concatenate([r[2][0] for r in out])
        lag = 3 - j
        for t in range(5):
            if t - lag >= 0:
                np.testing.assert_array_equal(got_v[t], ref_v[t - lag])
            else:  # comes from the stored history: same function of the raw history value
                (hv,), _ = _conv_run(sh, [unbf(raw[3 + t - lag])[None]], w_cur, np.zeros((3, C)))
                np.testing.assert_array_equal(got_v[t], hv[2][0, 0])
        np.testing.assert_array_equal(pool[0], raw[-3:])


def test_conv_weighted_sum_by_hand():
    # weights (0.5, -1, 2, 0.25), history (1, 2, -1), input 3 on every channel:
    # u = 0.5*1 - 1*2 + 2*(-1) + 0.25*3 = -2.75 (exact); v = u * sigmoid(u).
    sh = _shape(Hk=1, Hv=1, dk=16, dv=16, W=4)
    C = sh.channels
    w = np.tile([0.5, -1.0, 2.0, 0.25], (C, 1))
    hist = np.array([[1.0], [2.0], [-1.0]]) * np.ones((3, C))
    (r,), _ = _conv_run(sh, [np.full((1, C), 3.0)], w, hist)
    u = -2.75
    np.testing.assert_allclose(r[2], u / (1.0 + math.exp(-u)), rtol=1e-15)
    # reversed taps give a different value: the tap order is fixed
    (r2,), _ = _conv_run(sh, [np.full((1, C), 3.0)], w[:, ::-1].copy(), hist)
    u2 = 0.25 * 1 + 2 * 2 + (-1.0) * (-1) + 0.5 * 3  # = 6.75 with taps (0.25, 2, -1, 0.5)
    np.testing.assert_allclose(r2[2], u2 / (1.0 + math.exp(-u2)), rtol=1e-15)


def test_qk_unit_norm_and_direction():
    sh = _shape(Hk=3, Hv=3, dk=16, dv=16, W=4)
    C = sh.channels
    rng = np.random.default_rng(7)
    w = np.zeros((C, 4))
    w[:, 3] = 1.0
    x = rng.standard_normal((2, C))
    # a mirror layer whose V block receives every channel of x: its v output is the
    # pre-norm SiLU value of each channel, observable without any L2 norm
    shv = _shape(Hk=1, Hv=9, dk=16, dv=16, W=4)
    xm = np.zeros((2, shv.channels))
    xm[:, 32:] = x
    (r,), _ = _conv_run(sh, [x], w, np.zeros((3, C)))
    (rm,), _ = _conv_run(shv, [xm], np.eye(1, 4, 3).repeat(shv.channels, 0), np.zeros((3, shv.channels)))
    s_all = rm[2][0].reshape(2, C)
    s = s_all[:, :96].reshape(2, 2, 3, 16)  # [t][q|k][head][i]
    for t in range(2):
        for h in range(3):
            for which, vec, scale in ((0, r[0][0, t, h], 1 / 4.0), (1, r[1][0, t, h], 1.0)):
                sv = s[t, which, h]
                ns = np.linalg.norm(sv)
                n = np.linalg.norm(vec)
                # |q| sqrt(dk) = 1 and |k| = 1 up to eps/(2|s|^2)
                assert abs(n / scale - 1.0) <= 1e-6 / (2 * ns * ns) + 1e-14
                assert vec @ sv == pytest.approx(n * ns, rel=1e-13)  # parallel, same orientation
    # V channels carry the SiLU output with no norm
    np.testing.assert_array_equal(r[2][0].reshape(2, 48), s_all[:, 96:])


def test_l2_eps_sits_inside_the_root():
    # with |s|^2 comparable to eps the norm is |s| / sqrt(|s|^2 + eps), not |s| / max(|s|, eps)
    sh = _shape(Hk=1, Hv=1, dk=16, dv=16, W=4, q_scale=1.0)
    C = sh.channels
    w = np.zeros((C, 4))
    w[:, 3] = 1.0
    x = np.zeros((1, C))
    x[0, 0] = 2.0 ** -11  # silu(u) ~ u/2 ~ 2.4e-4: |s|^2 ~ 6e-8
    x[0, 16] = 2.0 ** -11
    (r,), _ = _conv_run(sh, [x], w, np.zeros((3, C)))
    # mirror through V to observe s
    shv = _shape(Hk=1, Hv=3, dk=16, dv=16, W=4)
    xm = np.zeros((1, shv.channels))
    xm[0, 32] = 2.0 ** -11
    (rm,), _ = _conv_run(shv, [xm], np.eye(1, 4, 3).repeat(shv.channels, 0), np.zeros((3, shv.channels)))
    s0 = rm[2][0, 0, 0, 0]
    assert np.linalg.norm(r[0][0, 0, 0]) == pytest.approx(s0 / math.sqrt(s0 * s0 + 1e-6), rel=1e-13)
    assert np.linalg.norm(r[0][0, 0, 0]) < 0.3
    # all-zero input: q = k = 0, no NaN
    (r0,), _ = _conv_run(sh, [np.zeros((1, C))], w, np.zeros((3, C)))
    assert np.all(r0[0] == 0) and np.all(r0[1] == 0)


def test_channel_layout_q_k_v_head_major():
    # step 6 splits Q | K | V sequentially, head-major inside each block.
    sh = _shape(Hk=2, Hv=4, dk=16, dv=16, W=4)
    C = sh.channels
    rng = np.random.default_rng(8)
    w = bf(rng.standard_normal((C, 4)))
    hist = rng.standard_normal((3, C))
    x = rng.standard_normal((1, C))
    (base,), _ = _conv_run(sh, [x], unbf(w), hist)

    def bumped(ch):
        x2 = x.copy()
        x2[0, ch] += 1.0
        (r,), _ = _conv_run(sh, [x2], unbf(w), hist)
        return [np.any(r[i] != base[i], axis=-1)[0, 0] for i in range(3)]

    dq, dk_, dv = bumped(1 * 16 + 3)           # Q channel of k-head 1
    assert list(dq) == [False, True] and not dk_.any() and not dv.any()
    dq, dk_, dv = bumped(2 * 16 + 0 * 16 + 5)  # K channel of k-head 0
    assert not dq.any() and list(dk_) == [True, False] and not dv.any()
    dq, dk_, dv = bumped(4 * 16 + 2 * 16 + 7)  # V channel of v-head 2
    assert not dq.any() and not dk_.any() and list(dv) == [False, False, True, False]


# --------------------------------------------------------------------------- step 8 (+ gate)
def test_gated_rmsnorm_properties():
    sh = _shape(Hk=1, Hv=3, dk=16, dv=16, rms_eps=1e-300)
    rng = np.random.default_rng(9)
    o = rng.standard_normal((2, 3, 16))
    z = bf(rng.standard_normal((2, 3, 16)) + 0.5)
    ones = bf(np.ones(16))
    out = oracle.gated_rmsnorm(sh, o, z, ones)
    zf = unbf(z)
    g = out / (zf / (1.0 + np.exp(-zf)))
    np.testing.assert_allclose(np.sqrt(np.mean(g * g, axis=-1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(g * np.sqrt(np.mean(o * o, -1, keepdims=True)), o, rtol=1e-13)
    # scale invariance in o, linearity in the per-column weight
    np.testing.assert_allclose(oracle.gated_rmsnorm(sh, 7.5 * o, z, ones), out, rtol=1e-13)
    w = np.ones(16)
    w[3] = 2.0
    w[9] = -0.5
    out_w = oracle.gated_rmsnorm(sh, o, z, bf(w))
    np.testing.assert_allclose(out_w, out * w, rtol=1e-15)
    # z = 0 closes the gate exactly
    assert np.all(oracle.gated_rmsnorm(sh, o, bf(np.zeros((2, 3, 16))), ones) == 0)


def test_gated_rmsnorm_eps():
    sh = _shape(Hk=1, Hv=1, dk=16, dv=16, rms_eps=1e-6)
    out = oracle.gated_rmsnorm(sh, np.zeros((1, 16)), bf(np.ones((1, 16))), bf(np.ones(16)))
    assert np.all(out == 0)
    o = np.full((1, 16), 1e-3)  # mean square 1e-6 = eps: RMS factor 1/sqrt(2e-6)
    out = oracle.gated_rmsnorm(sh, o, bf(np.full((1, 16), 30.0)), bf(np.ones(16)))
    np.testing.assert_allclose(out, 1e-3 / math.sqrt(2e-6) * 30.0, rtol=1e-12)


# --------------------------------------------------------------------------- whole step
def _random_problem(rng, Hk, Hv, dk, dv, W, B, T, P):
    sh = oracle.Shape(Hk, Hv, dk, dv, W)
    C = sh.channels
    d = dict(qkv=bf(rng.standard_normal((B, T, C))), a=bf(rng.standard_normal((B, T, Hv))),
             b=bf(rng.standard_normal((B, T, Hv))), z=bf(rng.standard_normal((B, T, Hv, dv))),
             conv_w=bf(0.5 * rng.standard_normal((C, W))),
             A_log=rng.uniform(-1, 1, Hv).astype(np.float32),
             dt_bias=(0.1 * rng.standard_normal(Hv)).astype(np.float32),
             norm_w=bf(1 + 0.05 * rng.standard_normal(dv)))
    conv_pool = bf(rng.standard_normal((P, W - 1, C)))
    state = 0.02 * rng.standard_normal((P, Hv, dk, dv))
    return sh, d, conv_pool, state


def _step(sh, d, conv_pool, state, slots, sl=slice(None)):
    return oracle.decode_step(sh, d["qkv"][sl], d["a"][sl], d["b"][sl], d["z"][sl], d["conv_w"],
                              d["A_log"], d["dt_bias"], d["norm_w"], conv_pool, state, slots)


def test_decode_step_composes_the_stages():
    rng = np.random.default_rng(10)
    sh, d, cp, st = _random_problem(rng, 2, 4, 16, 16, 4, B=2, T=3, P=3)
    slots = np.array([2, 0], np.int32)
    cp1, st1 = cp.copy(), st.copy()
    r = _step(sh, d, cp1, st1, slots)
    cp2, st2 = cp.copy(), st.copy()
    q, k, v = oracle.conv_update(sh, d["qkv"], d["conv_w"], cp2, slots)
    al, be = oracle.gate(sh, d["a"], d["b"], d["A_log"], d["dt_bias"])
    o = oracle.delta_rule(sh, q, k, v, al, be, st2, slots)
    out = oracle.gated_rmsnorm(sh, o, d["z"], d["norm_w"])
    for name, ref in (("q", q), ("k", k), ("v", v), ("alpha", al), ("beta", be), ("o", o), ("out", out)):
        np.testing.assert_array_equal(r[name], ref, err_msg=name)
    np.testing.assert_array_equal(cp1, cp2)
    np.testing.assert_array_equal(st1, st2)
    np.testing.assert_array_equal(cp1[1], cp[1])  # idle slot untouched
    np.testing.assert_array_equal(st1[1], st[1])


def test_multi_token_equals_sequential_single_tokens():
    rng = np.random.default_rng(11)
    sh, d, cp, st = _random_problem(rng, 2, 4, 16, 16, 4, B=2, T=5, P=2)
    slots = np.array([1, 0], np.int32)
    cpa, sta = cp.copy(), st.copy()
    ra = _step(sh, d, cpa, sta, slots)
    cpb, stb = cp.copy(), st.copy()
    outs = []
    for t in range(5):
        dt = {k: (v[:, t:t + 1] if k in ("qkv", "a", "b", "z") else v) for k, v in d.items()}
        outs.append(_step(sh, dt, cpb, stb, slots)["out"])
    np.testing.assert_array_equal(ra["out"], np.concatenate(outs, axis=1))
    np.testing.assert_array_equal(cpa, cpb)
    np.testing.assert_array_equal(sta, stb)


def test_gqa_equals_repeat_interleaved_keys():
    # Hv = 2 Hk with v-head h reading k-head h // 2 must equal an Hv = Hk layer whose
    # Q and K heads (inputs, conv weights and conv history) are repeat-interleaved.
    rng = np.random.default_rng(12)
    Hk, Hv, dk, dv, W, B, T = 2, 4, 16, 16, 4, 2, 2
    sh, d, cp, st = _random_problem(rng, Hk, Hv, dk, dv, W, B, T, P=2)
    slots = np.array([0, 1], np.int32)

    def dup(x, axis):  # channel axis: Q | K | V -> Q' | K' | V with heads repeated
        q, k, v = np.split(x, [Hk * dk, 2 * Hk * dk], axis=axis)
        rep = lambda y: np.repeat(np.stack(np.split(y, Hk, axis=axis), 0), 2, axis=0)  # noqa: E731
        q2 = np.concatenate(list(rep(q)), axis=axis)
        k2 = np.concatenate(list(rep(k)), axis=axis)
        return np.concatenate([q2, k2, v], axis=axis)

    sh2 = oracle.Shape(Hv, Hv, dk, dv, W)
    d2 = dict(d, qkv=dup(d["qkv"], 2), conv_w=dup(d["conv_w"], 0))
    cp2 = dup(cp, 2).copy()
    s1, s2 = st.copy(), st.copy()
    r1 = _step(sh, d, cp.copy(), s1, slots)
    r2 = _step(sh2, d2, cp2, s2, slots)
    np.testing.assert_array_equal(r1["out"], r2["out"])
    np.testing.assert_array_equal(s1, s2)


def test_gqa_head_map_by_perturbation():
    # a change in k-head 0's Q inputs reaches v-heads 0 and 1 only (h // G, not h % Hk)
    rng = np.random.default_rng(13)
    sh, d, cp, st = _random_problem(rng, 2, 4, 16, 16, 4, B=1, T=1, P=1)
    r0 = _step(sh, d, cp.copy(), st.copy(), [0])
    qkv = d["qkv"].copy()
    qkv[0, 0, 2] = bf(unbf(qkv[0, 0, 2:3]) + 1.0)[0]
    s1 = st.copy()
    r1 = _step(sh, dict(d, qkv=qkv), cp.copy(), s1, [0])
    changed = np.any(r1["out"] != r0["out"], axis=-1)[0, 0]
    assert list(changed) == [True, True, False, False]
    s0 = st.copy()
    _step(sh, d, cp.copy(), s0, [0])
    np.testing.assert_array_equal(s1, s0)  # q is read out only: the state does not see it


def test_sub_batch_equals_full_batch():
    # sequences are independent: the oracle on a subset (pool remapped) matches the
    # full run bit for bit, which is what the sampled full-size checks rely on.
    rng = np.random.default_rng(14)
    sh, d, cp, st = _random_problem(rng, 2, 4, 16, 16, 4, B=4, T=2, P=6)
    slots = np.array([5, 1, 3, 0], np.int32)
    full_cp, full_st = cp.copy(), st.copy()
    rf = _step(sh, d, full_cp, full_st, slots)
    pick = [1, 3]
    sub_cp, sub_st = cp[slots[pick]].copy(), st[slots[pick]].copy()
    rs = _step(sh, d, sub_cp, sub_st, np.arange(2, dtype=np.int32), sl=pick)
    np.testing.assert_array_equal(rs["out"], rf["out"][pick])
    np.testing.assert_array_equal(sub_st, full_st[slots[pick]])
    np.testing.assert_array_equal(sub_cp, full_cp[slots[pick]])


def test_round_bf16_is_correct_rne():
    x = np.array([1.0, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40, -3.0, 0.0, 2.0 ** -130,
                  65504.0, 1e-3])
    got = oracle.round_bf16(x)
    want = [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC040, 0x0000, 0x0008, 0x4780, 0x3A83]
    assert [int(g) for g in got] == want

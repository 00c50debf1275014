"""Pins for the oracle's speculative step (verify T drafted tokens, keep the state of
the accepted prefix): checks against properties the definition fixes, each through
a different route than the function itself (single-token steps, accept-then-rest,
the per-token factor form of the update).

Method source: the page "spark_model/forward/qwen3_5/linear_attention.rs" (the
decode step, steps 3 to 8) and, for the rollback to an accepted prefix, the page
"metrale_model_arch/glm5next_dsa/layer.rs" (lockstep check, rewind_to on a
rejected speculative draft).
"""
import numpy as np

import oracle
from gated_delta_rule_102_b200 import synth

bf = synth.to_bf16_bits


def _problem(rng, Hk=2, Hv=4, dk=16, dv=16, W=4, B=3, T=6, P=5):
    sh = oracle.Shape(Hk, Hv, dk, dv, W)
    C = sh.channels
    d = dict(qkv=bf(rng.normal(size=(B, T, C))), a=bf(rng.normal(size=(B, T, Hv))),
             b=bf(rng.normal(size=(B, T, Hv))), z=bf(rng.normal(size=(B, T, Hv, dv))),
             conv_w=bf(rng.normal(0, 0.5, size=(C, W))), A_log=rng.uniform(-1, 1, Hv).astype(np.float32),
             dt_bias=rng.normal(0, 0.1, Hv).astype(np.float32), norm_w=bf(1 + rng.normal(0, 0.05, dv)))
    cp = bf(rng.normal(size=(P, W - 1, C)))
    st = rng.normal(0, 0.02, size=(P, Hv, dk, dv))
    return sh, d, cp, st


def _tok(d, sl):
    return {k: (v[:, sl] if k in ("qkv", "a", "b", "z") else v) for k, v in d.items()}


def _step(sh, d, cp, st, slots, rows=slice(None)):
    x = {k: (v[rows] if k in ("qkv", "a", "b", "z") else v) for k, v in d.items()}
    return oracle.decode_step(sh, x["qkv"], x["a"], x["b"], x["z"], x["conv_w"], x["A_log"], x["dt_bias"],
                              x["norm_w"], cp, st, slots)


def _spec(sh, d, cp, st, slots, n):
    return oracle.speculative_step(sh, d["qkv"], d["a"], d["b"], d["z"], d["conv_w"], d["A_log"], d["dt_bias"],
                                   d["norm_w"], cp, st, slots, n)


SLOTS = np.array([4, 0, 2], np.int32)


def test_scores_every_drafted_token_whatever_is_accepted():
    rng = np.random.default_rng(21)
    sh, d, cp, st = _problem(rng)
    ref = _step(sh, d, cp.copy(), st.copy(), SLOTS)
    for n in ([0, 0, 0], [6, 6, 6], [1, 3, 5]):
        r = _spec(sh, d, cp.copy(), st.copy(), SLOTS, n)
        np.testing.assert_array_equal(r["out"], ref["out"])


def test_accepting_nothing_leaves_the_pools_bit_identical():
    rng = np.random.default_rng(22)
    sh, d, cp, st = _problem(rng)
    cp1, st1 = cp.copy(), st.copy()
    _spec(sh, d, cp1, st1, SLOTS, [0, 0, 0])
    np.testing.assert_array_equal(cp1, cp)
    np.testing.assert_array_equal(st1, st)


def test_accepting_everything_is_the_full_step():
    rng = np.random.default_rng(23)
    sh, d, cp, st = _problem(rng)
    cp1, st1, cp2, st2 = cp.copy(), st.copy(), cp.copy(), st.copy()
    _spec(sh, d, cp1, st1, SLOTS, [6, 6, 6])
    _step(sh, d, cp2, st2, SLOTS)
    np.testing.assert_array_equal(cp1, cp2)
    np.testing.assert_array_equal(st1, st2)


def test_accepted_prefix_equals_that_many_single_token_steps():
    rng = np.random.default_rng(24)
    sh, d, cp, st = _problem(rng)
    n = [2, 0, 5]
    cp1, st1 = cp.copy(), st.copy()
    _spec(sh, d, cp1, st1, SLOTS, n)
    cp2, st2 = cp.copy(), st.copy()
    for i, ni in enumerate(n):
        for t in range(ni):
            _step(sh, _tok(d, slice(t, t + 1)), cp2, st2, SLOTS[i:i + 1], rows=slice(i, i + 1))
    np.testing.assert_array_equal(cp1, cp2)
    np.testing.assert_array_equal(st1, st2)
    idle = [1, 3]  # slots no sequence names
    np.testing.assert_array_equal(cp1[idle], cp[idle])
    np.testing.assert_array_equal(st1[idle], st[idle])


def test_accept_a_prefix_then_the_rest_equals_accepting_all():
    rng = np.random.default_rng(25)
    sh, d, cp, st = _problem(rng, B=1)
    slots = np.array([3], np.int32)
    for n in range(7):
        cp1, st1 = cp.copy(), st.copy()
        _spec(sh, d, cp1, st1, slots, [n])
        if n < 6:
            _step(sh, _tok(d, slice(n, 6)), cp1, st1, slots)
        cp2, st2 = cp.copy(), st.copy()
        _step(sh, d, cp2, st2, slots)
        np.testing.assert_array_equal(cp1, cp2)
        np.testing.assert_allclose(st1, st2, rtol=0, atol=1e-15)


def test_state_of_the_prefix_is_the_replay_of_per_token_factors():
    # The state after n tokens is S_n = alpha_t S_{t-1} + k_t delta_t^T applied in order,
    # with delta_t = beta_t (v_t - alpha_t S_{t-1}^T k_t): the factor form a commit pass
    # replays. k, v, alpha, beta are the decode step's own intermediates.
    rng = np.random.default_rng(26)
    sh, d, cp, st = _problem(rng, B=1)
    slots = np.array([1], np.int32)
    full = _step(sh, d, cp.copy(), st.copy(), slots)
    G = sh.num_v_heads // sh.num_k_heads
    for n in (1, 4, 6):
        cp1, st1 = cp.copy(), st.copy()
        _spec(sh, d, cp1, st1, slots, [n])
        for h in range(sh.num_v_heads):
            S = st[1, h].copy()
            for t in range(n):
                k = full["k"][0, t, h // G]
                al, be, v = full["alpha"][0, t, h], full["beta"][0, t, h], full["v"][0, t, h]
                delta = be * (v - al * (S.T @ k))
                S = al * S + np.outer(k, delta)
            np.testing.assert_allclose(st1[1, h], S, rtol=0, atol=1e-13)

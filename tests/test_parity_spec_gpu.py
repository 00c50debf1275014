"""GPU parity of speculative decoding through the C ABI: gdn_spec_verify scores T
drafted tokens without touching the pools, gdn_spec_commit keeps the accepted
prefix. Checked against the oracle's speculative step (outputs of all T tokens,
pools advanced by n_accept[b] tokens) for every sequence, over two rounds in a row
(the second verifies from the state the first committed).

Bars: outputs as for the decode step (fp32 within 2e-3 absolute, bf16 the RNE of
it); the verify call leaves both pools bit-identical; after the commit the conv
history of every sequence is bit-exact and its state within 1e-4 (per slot and
head, relative to the head's largest entry); the recorded keys and decays match the
oracle's normalised keys and decays."""
import zlib

import numpy as np
import pytest
import torch

import gated_delta_rule_102_b200 as gdn
import oracle
from gated_delta_rule_102_b200 import synth
from gdn_harness import DeviceRun, OracleRun, bf16_host, compare_out, compare_state

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["tiny_d16"]


def wl_of(name, Hk, Hv, dk, dv, W, B, T, P, gate_mode="normal"):
    return BASE.replace(name=name, num_k_heads=Hk, num_v_heads=Hv, head_k_dim=dk, head_v_dim=dv, conv_width=W,
                        batch=B, tokens=T, pool_slots=P, steps=2, seed=zlib.crc32(name.encode()) % 10000,
                        slot_mode="sample", state_std=0.02, gate_mode=gate_mode)


def accept_counts(B, T, rnd, seed):
    """Per sequence 0, 1, T/2, T or a draw in between (every kind present when B >= 4)."""
    rng = np.random.default_rng(seed * 31 + rnd)
    kinds = [0, min(1, T), T // 2, T]
    n = [kinds[(i + rnd) % 4] if i < 4 else int(rng.integers(0, T + 1)) for i in range(B)]
    return np.array(n, np.int32)


class SpecBuffers:
    def __init__(self, wl):
        B, T = wl.batch, wl.tokens
        self.out = torch.empty(B, T, wl.num_v_heads, wl.head_v_dim, dtype=torch.bfloat16, device="cuda")
        self.out32 = torch.empty(B, T, wl.num_v_heads, wl.head_v_dim, dtype=torch.float32, device="cuda")
        self.k = torch.empty(B, T, wl.num_k_heads, wl.head_k_dim, dtype=torch.float32, device="cuda")
        self.delta = torch.empty(B, T, wl.num_v_heads, wl.head_v_dim, dtype=torch.float32, device="cuda")
        self.alpha = torch.empty(B, T, wl.num_v_heads, dtype=torch.float32, device="cuda")


def verify(g, x, sb):
    gdn.gdn_spec_verify(g.cfg, x["qkv"], x["a"], x["b"], x["z"], g.conv_w, g.A_log, g.dt_bias, g.norm_w, g.conv,
                        g.state, g.slots, sb.out, sb.k, sb.delta, sb.alpha, sb.out32, g.err)


def commit(g, x, sb, n):
    gdn.gdn_spec_commit(g.cfg, torch.from_numpy(n).cuda(), x["qkv"], g.conv, g.state, g.slots, sb.k, sb.delta,
                        sb.alpha, g.err)


def run_rounds(wl, rounds=2):
    g = DeviceRun(wl)
    rows = list(range(wl.batch))
    o = OracleRun(wl, rows)
    sb = SpecBuffers(wl)
    idle = sorted(set(range(wl.pool_slots)) - set(g.slots_np.tolist()))
    pool_idle = g.state[idle].clone() if idle else None
    for rnd in range(rounds):
        x = g.inputs(rnd)
        conv0, state0 = g.conv.clone(), g.state.clone()
        verify(g, x, sb)
        torch.cuda.synchronize()
        assert torch.equal(g.conv, conv0) and torch.equal(g.state, state0), "verify wrote a pool"
        n = accept_counts(wl.batch, wl.tokens, rnd, wl.seed)
        xo = synth.step_inputs(wl, rnd, rows=rows)
        w = o.w
        r = oracle.speculative_step(o.shape, xo["qkv"], xo["a"], xo["b"], xo["z"], w["conv_w"], w["A_log"],
                                    w["dt_bias"], w["norm_w"], o.conv, o.state, o.local, n)
        compare_out(sb.out, sb.out32, r["out"], rows, f"{wl.name} round {rnd} verify")
        np.testing.assert_allclose(sb.k.cpu().numpy(), r["k"], rtol=0, atol=2e-6)
        # alpha = exp(g): an error e in g is a relative error e in alpha, and g carries a few
        # fp32 roundings of its own size, so the bound grows with |g| = -ln(alpha)
        ga, ra = sb.alpha.cpu().numpy().astype(np.float64), r["alpha"]
        lim = 1e-6 * (1.0 + np.abs(np.log(np.maximum(ra, 1e-300)))) * ra + 1e-37
        assert np.all(np.abs(ga - ra) <= lim), f"{wl.name}: recorded decays"
        commit(g, x, sb, n)
        torch.cuda.synchronize()
        assert int(g.err.item()) == 0
        compare_state(g.state, o.state, o.slot_ids, f"{wl.name} round {rnd} commit")
        np.testing.assert_array_equal(bf16_host(g.conv)[o.slot_ids], o.conv)
    if idle:
        assert torch.equal(g.state[idle], pool_idle)
    return g, o


def test_spec_multitoken_b32_t16_every_sequence():
    # the multi-token workload's shape (B=32 x T=16 drafted tokens, Hk=16, Hv=32, dk=dv=128)
    run_rounds(synth.WORKLOADS["multitoken_b32_t16"].replace(pool_slots=40, slot_mode="sample"))


SHAPES = [
    # name                  Hk Hv  dk   dv  W  B  T  P   gate
    ("spec_d16_t5", 1, 2, 16, 16, 4, 3, 5, 4, "normal"),
    ("spec_dk64_dv32_g4_t3", 2, 8, 64, 32, 3, 4, 3, 6, "normal"),
    ("spec_t1", 2, 4, 32, 32, 2, 4, 1, 5, "normal"),
    ("spec_w8_t7", 2, 4, 32, 64, 8, 4, 7, 5, "normal"),
    ("spec_wide_t16", 2, 4, 128, 128, 4, 4, 16, 5, "decay_wide"),
    ("spec_d128_t1", 2, 4, 128, 128, 4, 3, 1, 5, "normal"),  # one drafted token, the chunked kernel
]


@pytest.mark.parametrize("spec", SHAPES, ids=[s[0] for s in SHAPES])
def test_spec_shapes(spec):
    name, Hk, Hv, dk, dv, W, B, T, P, gate = spec
    run_rounds(wl_of(name, Hk, Hv, dk, dv, W, B, T, P, gate_mode=gate))


def test_commit_nothing_leaves_pools_bit_identical_and_bad_counts_are_flagged():
    wl = wl_of("spec_flags", 2, 4, 64, 64, 4, 4, 6, 6)
    g = DeviceRun(wl)
    sb = SpecBuffers(wl)
    x = g.inputs(0)
    verify(g, x, sb)
    conv0, state0 = g.conv.clone(), g.state.clone()
    commit(g, x, sb, np.zeros(4, np.int32))
    torch.cuda.synchronize()
    assert torch.equal(g.conv, conv0) and torch.equal(g.state, state0) and int(g.err.item()) == 0
    # sequences 1 and 2 ask for counts outside [0, T]: skipped and flagged; 0 and 3 commit
    commit(g, x, sb, np.array([6, 7, -1, 2], np.int32))
    torch.cuda.synchronize()
    assert int(g.err.item()) == gdn.GDN_DEVICE_ERR_SEQLEN
    s = g.slots_np
    for i in (1, 2):
        assert torch.equal(g.state[int(s[i])], state0[int(s[i])])
        assert torch.equal(g.conv[int(s[i])], conv0[int(s[i])])
    for i in (0, 3):
        assert not torch.equal(g.state[int(s[i])], state0[int(s[i])])

"""GPU parity across shapes and edge cases: head dims 16..128 with dk != dv, GQA
ratios 1..8 (including 3, a non power of two cluster), conv widths 2..8, T = 1..16,
ragged batches, sparse pools; the three stage entry points one by one; bad slots;
empty batches; split runs; determinism."""
import zlib

import numpy as np
import pytest
import torch

import gated_delta_rule_102_b200 as gdn
import oracle
from gated_delta_rule_102_b200 import synth
from gdn_harness import (DeviceRun, OracleRun, bf16_dev, bf16_host, compare_out, compare_state, conv_pool_reference,
                         f32_dev)

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["tiny_d16"]


def wl_of(name, Hk, Hv, dk, dv, W, B, T, P, steps, seed, slot_mode="sample", std=0.02, gate_mode="normal"):
    if slot_mode == "permutation":
        P = B
    return BASE.replace(name=name, num_k_heads=Hk, num_v_heads=Hv, head_k_dim=dk, head_v_dim=dv, conv_width=W,
                        batch=B, tokens=T, pool_slots=P, steps=steps, seed=seed, slot_mode=slot_mode,
                        state_std=std, gate_mode=gate_mode)


SHAPES = [
    # name            Hk Hv  dk   dv  W  B  T  P  steps
    ("dk64_dv128_g2", 2, 4, 64, 128, 4, 3, 1, 5, 3),
    ("dk128_dv32_g8", 1, 8, 128, 32, 3, 2, 2, 3, 3),
    ("dk32_dv64_g1", 3, 3, 32, 64, 2, 5, 4, 7, 2),
    ("dk16_dv128_g3", 2, 6, 16, 128, 4, 2, 3, 2, 3),
    ("dk128_g4_t16", 4, 16, 128, 128, 4, 2, 16, 3, 2),
    ("d16_t16", 1, 2, 16, 16, 4, 3, 16, 4, 2),
    ("w8_t5", 2, 4, 32, 32, 8, 2, 5, 2, 3),
    ("w2_t1_b1", 16, 32, 128, 128, 2, 1, 1, 1, 3),
    ("dk64_dv16_g4_t7", 2, 8, 64, 16, 3, 4, 7, 9, 2),
    ("b33_ragged", 2, 4, 128, 64, 4, 33, 1, 40, 2),
    ("dk64_dv128_g8_t16", 1, 8, 64, 128, 4, 2, 16, 2, 2),
]


@pytest.mark.parametrize("spec", SHAPES, ids=[s[0] for s in SHAPES])
def test_fused_matches_oracle(spec, gate_mode="normal"):
    name, Hk, Hv, dk, dv, W, B, T, P, steps = spec
    wl = wl_of(name, Hk, Hv, dk, dv, W, B, T, P, steps, seed=zlib.crc32(name.encode()) % 10000,
               gate_mode=gate_mode)
    g = DeviceRun(wl)
    rows = list(range(B))
    o = OracleRun(wl, rows)
    pool0 = g.state.clone()
    for s in range(steps):
        out, out32 = g.step(g.inputs(s))
        r = o.step(s)
        compare_out(out, out32, r["out"], rows, f"{name} step {s}")
    torch.cuda.synchronize()
    assert int(g.err.item()) == 0
    compare_state(g.state, o.state, o.slot_ids, name)
    np.testing.assert_array_equal(bf16_host(g.conv), conv_pool_reference(wl, steps))
    idle = sorted(set(range(P)) - set(g.slots_np.tolist()))
    if idle:
        idx = torch.tensor(idle, device="cuda")
        assert torch.equal(g.state[idx], pool0[idx])


# Decays from 1 down to fp32 underflow (exp(g) = 2^-u, u up to 48, and 2^-200): the
# multi-token kernel carries the decay as a running scale and must fold it into the
# state before it underflows; the single-token kernels multiply directly.
WIDE_DECAY_SHAPES = [
    # name               Hk Hv  dk   dv  W   B  T   P  steps
    ("wide_t16", 2, 4, 128, 128, 4, 3, 16, 4, 2),
    ("wide_t5_dk16_dv32", 1, 2, 16, 32, 3, 2, 5, 3, 2),
    ("wide_t1", 2, 4, 64, 64, 4, 3, 1, 5, 2),
    ("wide_t1_persistent", 4, 8, 128, 128, 4, 40, 1, 48, 2),
]


@pytest.mark.parametrize("spec", WIDE_DECAY_SHAPES, ids=[s[0] for s in WIDE_DECAY_SHAPES])
def test_wide_decay_matches_oracle(spec):
    test_fused_matches_oracle(spec, gate_mode="decay_wide")


# Single-token launches with many (sequence, k-head) groups take the persistent
# pipelined kernel (at least two groups per co-resident cluster).
PERSISTENT_SHAPES = [
    # name              Hk Hv   dk   dv  W    B  T    P  steps
    ("p_d128_g2", 4, 8, 128, 128, 4, 40, 1, 48, 3),
    ("p_d128_g1_w2", 8, 8, 128, 128, 2, 40, 1, 44, 2),
    ("p_dk128_dv64_g4", 2, 8, 128, 64, 4, 80, 1, 80, 2),
    ("p_dk64_dv128_g8_w3", 1, 8, 64, 128, 3, 100, 1, 101, 2),
    ("p_dk128_dv32_g2_w3", 4, 8, 128, 32, 3, 48, 1, 50, 3),
    ("p_dk32_dv128_g4", 2, 8, 32, 128, 4, 80, 1, 90, 2),
]


@pytest.mark.parametrize("spec", PERSISTENT_SHAPES, ids=[s[0] for s in PERSISTENT_SHAPES])
def test_persistent_path_matches_oracle(spec):
    test_fused_matches_oracle(spec)


def test_persistent_path_bad_slot():
    wl = wl_of("p_badslot", 4, 8, 128, 128, 4, 40, 1, 40, 1, seed=21, slot_mode="permutation")
    g = DeviceRun(wl)
    slots = g.slots_np.copy()
    slots[17] = 40  # outside the 40-slot pool
    g.slots = torch.from_numpy(slots).cuda()
    state0, conv0 = g.state.clone(), g.conv.clone()
    x = g.inputs(0)
    shape = (40, 1, 8, 128)
    out = torch.full(shape, 3.0, dtype=torch.bfloat16, device="cuda")
    out32 = torch.full(shape, 3.0, device="cuda")
    gdn.gdn_decode_step(g.cfg, x["qkv"], x["a"], x["b"], x["z"], g.conv_w, g.A_log, g.dt_bias, g.norm_w,
                        g.conv, g.state, g.slots, out, out32, g.err, g.workspace)
    torch.cuda.synchronize()
    assert int(g.err.item()) == gdn.GDN_DEVICE_ERR_SLOT_RANGE
    assert torch.all(out32[17] == 3.0)
    assert int(g.workspace.abs().sum().item()) == 0
    skipped = int(g.slots_np[17])  # the slot sequence 17 would have used: nobody touched it
    assert torch.equal(g.state[skipped], state0[skipped]) and torch.equal(g.conv[skipped], conv0[skipped])
    rows = [0, 16, 18, 39]
    o = OracleRun(wl, rows)
    r = o.step(0)
    compare_out(out, out32, r["out"], rows, "persistent rows beside a bad slot")
    compare_state(g.state, o.state, o.slot_ids, "persistent rows beside a bad slot")


def _stage_problem(seed=5, Hk=2, Hv=4, dk=64, dv=128, W=4, B=3, T=3, P=4):
    wl = wl_of("stages", Hk, Hv, dk, dv, W, B, T, P, 1, seed)
    return wl, DeviceRun(wl), synth.step_inputs(wl, 0)


def test_conv_stage_matches_oracle():
    wl, g, x = _stage_problem()
    B, T = wl.batch, wl.tokens
    q = torch.empty(B, T, wl.num_k_heads, wl.head_k_dim, device="cuda")
    k = torch.empty_like(q)
    v = torch.empty(B, T, wl.num_v_heads, wl.head_v_dim, device="cuda")
    gdn.gdn_conv_update(g.cfg, bf16_dev(x["qkv"]), g.conv_w, g.conv, g.slots, q, k, v, g.err)
    pool = synth.initial_conv_state(wl)
    w = synth.weights(wl)
    rq, rk, rv = oracle.conv_update(oracle.Shape.of(wl), x["qkv"], w["conv_w"], pool, g.slots_np)
    torch.cuda.synchronize()
    np.testing.assert_allclose(q.cpu().numpy(), rq, rtol=0, atol=2e-6)
    np.testing.assert_allclose(k.cpu().numpy(), rk, rtol=0, atol=2e-6)
    np.testing.assert_allclose(v.cpu().numpy(), rv, rtol=2e-6, atol=2e-6)
    np.testing.assert_array_equal(bf16_host(g.conv), pool)


def test_recurrent_stage_matches_oracle():
    wl, g, x = _stage_problem(seed=6, T=5)
    B, T = wl.batch, wl.tokens
    rng = np.random.default_rng(0)
    q = rng.standard_normal((B, T, wl.num_k_heads, wl.head_k_dim)).astype(np.float32)
    k = rng.standard_normal(q.shape).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, wl.num_v_heads, wl.head_v_dim)).astype(np.float32)
    o = torch.empty(B, T, wl.num_v_heads, wl.head_v_dim, device="cuda")
    gdn.gdn_recurrent_step(g.cfg, f32_dev(q), f32_dev(k), f32_dev(v), bf16_dev(x["a"]), bf16_dev(x["b"]),
                           g.A_log, g.dt_bias, g.state, g.slots, o, g.err)
    w = synth.weights(wl)
    sh = oracle.Shape.of(wl)
    al, be = oracle.gate(sh, x["a"], x["b"], w["A_log"], w["dt_bias"])
    st = synth.initial_state(wl).astype(np.float64)
    ro = oracle.delta_rule(sh, q, k, v, al, be, st, g.slots_np)
    torch.cuda.synchronize()
    scale = np.abs(ro).max()
    assert np.abs(o.cpu().numpy() - ro).max() <= 1e-5 * scale
    compare_state(g.state, st[g.slots_np], [int(s) for s in g.slots_np], "recurrent stage")


def test_gated_rmsnorm_stage_matches_oracle():
    wl, g, x = _stage_problem(seed=7)
    rng = np.random.default_rng(1)
    o = rng.standard_normal((wl.batch, wl.tokens, wl.num_v_heads, wl.head_v_dim)).astype(np.float32)
    out = torch.empty(o.shape, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(o.shape, dtype=torch.float32, device="cuda")
    gdn.gdn_gated_rmsnorm(g.cfg, f32_dev(o), bf16_dev(x["z"]), g.norm_w, out, out32)
    ref = oracle.gated_rmsnorm(oracle.Shape.of(wl), o, x["z"], synth.weights(wl)["norm_w"])
    compare_out(out, out32, ref, list(range(wl.batch)), "gated rmsnorm")
    assert np.abs(out32.cpu().numpy() - ref).max() < 1e-5


def test_fused_equals_stage_chain():
    wl, g, x = _stage_problem(seed=8, T=2)
    g2 = DeviceRun(wl)
    B, T = wl.batch, wl.tokens
    out, out32 = g.step({k: bf16_dev(v) for k, v in x.items()})
    q = torch.empty(B, T, wl.num_k_heads, wl.head_k_dim, device="cuda")
    k = torch.empty_like(q)
    v = torch.empty(B, T, wl.num_v_heads, wl.head_v_dim, device="cuda")
    gdn.gdn_conv_update(g2.cfg, bf16_dev(x["qkv"]), g2.conv_w, g2.conv, g2.slots, q, k, v)
    o = torch.empty_like(v)
    gdn.gdn_recurrent_step(g2.cfg, q, k, v, bf16_dev(x["a"]), bf16_dev(x["b"]), g2.A_log, g2.dt_bias,
                           g2.state, g2.slots, o)
    out2 = torch.empty_like(out)
    out2_32 = torch.empty_like(out32)
    gdn.gdn_gated_rmsnorm(g2.cfg, o, bf16_dev(x["z"]), g2.norm_w, out2, out2_32)
    torch.cuda.synchronize()
    assert (out32 - out2_32).abs().max().item() < 1e-4
    assert torch.equal(g.conv, g2.conv)
    assert ((g.state - g2.state).abs().max() / g.state.abs().max()).item() < 1e-5


def test_out_of_range_slot_is_skipped_and_flagged():
    wl = wl_of("badslot", 2, 4, 32, 32, 4, 3, 1, 4, 1, seed=9)
    g = DeviceRun(wl)
    g.slots = torch.tensor([1, 7, 3], dtype=torch.int32, device="cuda")  # 7 is outside the 4-slot pool
    g.slots_np = g.slots.cpu().numpy()
    state0, conv0 = g.state.clone(), g.conv.clone()
    x = g.inputs(0)
    shape = (3, 1, 4, 32)
    out = torch.full(shape, 7.0, dtype=torch.bfloat16, device="cuda")
    out32 = torch.full(shape, 7.0, device="cuda")
    gdn.gdn_decode_step(g.cfg, x["qkv"], x["a"], x["b"], x["z"], g.conv_w, g.A_log, g.dt_bias, g.norm_w,
                        g.conv, g.state, g.slots, out, out32, g.err)
    torch.cuda.synchronize()
    assert int(g.err.item()) == gdn.GDN_DEVICE_ERR_SLOT_RANGE
    assert torch.all(out32[1] == 7.0) and torch.all(out[1].float() == 7.0)
    for s in (0, 2):  # untouched slots keep their bytes
        assert torch.equal(g.state[s], state0[s]) and torch.equal(g.conv[s], conv0[s])
    # the valid sequences were computed as usual
    o = OracleRun(wl.replace(pool_slots=4), [0, 2], state0=state0.cpu().numpy())
    o.slot_ids = [1, 3]
    o.state = state0.cpu().numpy()[[1, 3]].astype(np.float64)
    r = o.step(0)
    compare_out(out, out32, r["out"], [0, 2], "valid rows beside a bad slot")
    # and the stage kernels flag it too
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = torch.empty(3, 1, 2, 32, device="cuda")
    gdn.gdn_conv_update(g.cfg, x["qkv"], g.conv_w, g.conv, g.slots, q, q.clone(),
                        torch.empty(3, 1, 4, 32, device="cuda"), err)
    torch.cuda.synchronize()
    assert int(err.item()) == gdn.GDN_DEVICE_ERR_SLOT_RANGE


def test_empty_batch_is_a_no_op_on_device():
    wl = wl_of("empty", 2, 4, 32, 32, 4, 2, 1, 2, 1, seed=10)
    g = DeviceRun(wl)
    st, cv = g.state.clone(), g.conv.clone()
    e = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device="cuda")  # noqa: E731
    gdn.gdn_decode_step(g.cfg, e(0, 1, wl.channels), e(0, 1, 4), e(0, 1, 4), e(0, 1, 4, 32), g.conv_w, g.A_log,
                        g.dt_bias, g.norm_w, g.conv, g.state, e(0, dt=torch.int32), e(0, 1, 4, 32))
    torch.cuda.synchronize()
    assert torch.equal(g.state, st) and torch.equal(g.conv, cv)


def test_split_run_resumes_bit_identically():
    # N steps, pools copied to the host and back into fresh buffers, M more steps:
    # the same bits as N + M steps in one go (the pools are the whole resumable state).
    wl = wl_of("resume", 2, 4, 64, 64, 4, 4, 2, 6, 6, seed=11)
    a = DeviceRun(wl)
    for s in range(6):
        out_a, _ = a.step(a.inputs(s))
    b = DeviceRun(wl)
    for s in range(3):
        b.step(b.inputs(s))
    state_host, conv_host = b.state.cpu(), b.conv.cpu()
    c = DeviceRun(wl)
    c.state.copy_(state_host.cuda())
    c.conv.copy_(conv_host.cuda())
    for s in range(3, 6):
        out_c, _ = c.step(c.inputs(s))
    torch.cuda.synchronize()
    assert torch.equal(a.state, c.state) and torch.equal(a.conv, c.conv) and torch.equal(out_a, out_c)


def test_deterministic():
    wl = wl_of("det", 2, 4, 128, 128, 4, 8, 1, 8, 1, seed=12, slot_mode="permutation")
    a, b = DeviceRun(wl), DeviceRun(wl)
    x = a.inputs(0)
    oa, oa32 = a.step(x)
    ob, ob32 = b.step(x)
    torch.cuda.synchronize()
    assert torch.equal(oa, ob) and torch.equal(oa32, ob32) and torch.equal(a.state, b.state)


@pytest.mark.parametrize("name", ["batch64_small", "tiny_d16", "multitoken"])
def test_step_replays_from_a_cuda_graph(name):
    # a decode engine captures the step once and replays it: the replay must give the
    # same bits as eager launches (both the persistent and the per-tile kernels)
    base = {"batch64_small": synth.WORKLOADS["batch64"].replace(batch=40, pool_slots=40, num_k_heads=4,
                                                                 num_v_heads=8),
            "tiny_d16": synth.WORKLOADS["tiny_d16"],
            "multitoken": synth.WORKLOADS["multitoken_b32_t16"].replace(batch=4, pool_slots=4)}[name]
    eager, graphed = DeviceRun(base), DeviceRun(base)
    xs = [eager.inputs(s) for s in range(3)]
    outs_e = [eager.step(x)[1].clone() for x in xs]
    graphed.step(xs[0])  # first call on the device outside the capture (one-time set-up)
    graphed.state.copy_(DeviceRun(base).state)
    graphed.conv.copy_(DeviceRun(base).conv)
    shape = (base.batch, base.tokens, base.num_v_heads, base.head_v_dim)
    outs = [torch.empty(shape, device="cuda") for _ in xs]
    outb = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        for x, o in zip(xs, outs):
            gdn.gdn_decode_step(graphed.cfg, x["qkv"], x["a"], x["b"], x["z"], graphed.conv_w, graphed.A_log,
                                graphed.dt_bias, graphed.norm_w, graphed.conv, graphed.state, graphed.slots, outb, o,
                                graphed.err, graphed.workspace)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs_e, outs):
        assert torch.equal(a, b)
    assert torch.equal(eager.state, graphed.state) and torch.equal(eager.conv, graphed.conv)
    assert int(graphed.err.item()) == 0


@pytest.mark.parametrize("spec", [PERSISTENT_SHAPES[0], PERSISTENT_SHAPES[2]], ids=["g2", "g4"])
def test_dynamic_and_static_schedules_agree(spec):
    # the workspace only changes which SM takes which sequence: the same bits come out,
    # and the workspace is left zeroed for the next call
    name, Hk, Hv, dk, dv, W, B, T, P, steps = spec
    wl = wl_of(name, Hk, Hv, dk, dv, W, B, T, P, steps, seed=77)
    dyn, sta = DeviceRun(wl, dynamic=True), DeviceRun(wl, dynamic=False)
    for s in range(steps):
        x = dyn.inputs(s)
        od, od32 = dyn.step(x)
        os_, os32 = sta.step(x)
        torch.cuda.synchronize()
        assert torch.equal(od32, os32) and torch.equal(od, os_)
        assert int(dyn.workspace.abs().sum().item()) == 0
    assert torch.equal(dyn.state, sta.state) and torch.equal(dyn.conv, sta.conv)


# Launches of different token counts on the same pools (a chunk of several tokens, then
# single tokens, and so on) must act like the same tokens run in order. The kernels
# for one token and for several differ, and a launch may begin while the previous one
# drains (programmatic dependent launch): every read of a pool waits for that grid.
MIXED = [
    # name          Hk Hv   dk   dv  W   B   P   token counts of the launches
    ("mixed_small", 2, 4, 128, 128, 4, 3, 5, [5, 1, 16, 1, 1, 3, 2]),        # cluster kernel for T = 1
    ("mixed_persist", 4, 8, 128, 128, 4, 40, 43, [1, 4, 1, 1, 16, 1]),      # persistent kernel for T = 1
    ("mixed_w3_dv64", 2, 8, 64, 64, 3, 5, 6, [2, 1, 7, 1]),
]


@pytest.mark.parametrize("spec", MIXED, ids=[m[0] for m in MIXED])
def test_mixed_token_counts_share_pools(spec):
    name, Hk, Hv, dk, dv, W, B, P, counts = spec
    wl1 = wl_of(name, Hk, Hv, dk, dv, W, B, 1, P, len(counts), seed=zlib.crc32(name.encode()) % 10000)
    g = DeviceRun(wl1)
    rows = sorted({0, B // 2, B - 1})
    o = OracleRun(wl1, rows)
    pool0 = g.state.clone()
    for i, T in enumerate(counts):
        wl = wl1.replace(tokens=T)
        x = {k: bf16_dev(v) for k, v in synth.step_inputs(wl, i).items()}
        shape = (B, T, Hv, dv)
        out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        out32 = torch.empty(shape, dtype=torch.float32, device="cuda")
        gdn.gdn_decode_step(g.cfg, x["qkv"], x["a"], x["b"], x["z"], g.conv_w, g.A_log, g.dt_bias, g.norm_w, g.conv,
                            g.state, g.slots, out, out32, g.err, g.workspace)
        xr = synth.step_inputs(wl, i, rows=rows)
        w = o.w
        r = oracle.decode_step(o.shape, xr["qkv"], xr["a"], xr["b"], xr["z"], w["conv_w"], w["A_log"], w["dt_bias"],
                               w["norm_w"], o.conv, o.state, o.local)
        compare_out(out, out32, r["out"], rows, f"{name} launch {i} (T={T})")
    torch.cuda.synchronize()
    assert int(g.err.item()) == 0
    compare_state(g.state, o.state, o.slot_ids, name)
    np.testing.assert_array_equal(bf16_host(g.conv)[o.slot_ids], o.conv)
    idle = sorted(set(range(P)) - set(g.slots_np.tolist()))
    if idle:
        idx = torch.tensor(idle, device="cuda")
        assert torch.equal(g.state[idx], pool0[idx])

"""GPU parity of the chunked tensor-core form of the multi-token step (dk = dv = 128,
T = 2..16 tokens per launch): the single-token recurrence unrolled over the launch's
tokens, its two contractions on tcgen05 in split tf32. Checked against the oracle's
token-by-token step (outputs, states, conv pools) on the cases the chunk form has to
get right beyond the shared tests: conv widths whose history outlives the launch's
tokens (W - 1 > T), one v-head per k-head and odd GQA ratios, many groups per CTA
(double-buffered operand tiles, the state ring wrapping), large state entries (the
low tf32 parts carry real weight), decays down to underflow, the device batch count
under graph replay, and bit-for-bit determinism."""
import zlib

import numpy as np
import pytest
import torch

import gated_delta_rule_102_b200 as gdn
from gated_delta_rule_102_b200 import synth
from gdn_harness import DeviceRun, OracleRun, bf16_host, compare_out, compare_state, conv_pool_reference

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["tiny_d16"]


def wl_of(name, Hk, Hv, W, B, T, P, steps, std=0.02, gate_mode="normal"):
    return BASE.replace(name=name, num_k_heads=Hk, num_v_heads=Hv, head_k_dim=128, head_v_dim=128, conv_width=W,
                        batch=B, tokens=T, pool_slots=P, steps=steps, seed=zlib.crc32(name.encode()) % 10000,
                        slot_mode="sample", state_std=std, gate_mode=gate_mode)


CASES = [
    # name                Hk  Hv  W   B   T   P  steps  state std  gates
    ("c_g1_w2_t2", 4, 4, 2, 3, 2, 5, 3, 0.02, "normal"),
    ("c_g2_w8_t3", 2, 4, 8, 3, 3, 4, 3, 0.02, "normal"),      # history of 7 rows, 3 tokens per launch
    ("c_g3_w3_t9", 2, 6, 3, 2, 9, 3, 2, 0.02, "normal"),
    ("c_g2_t16_many_groups", 16, 32, 4, 20, 5, 24, 2, 0.02, "normal"),  # 320 groups: 2-3 per CTA
    ("c_big_state_t16", 2, 4, 4, 3, 16, 4, 2, 1.0, "normal"),
    ("c_wide_decay_t7", 2, 4, 4, 3, 7, 4, 2, 0.02, "decay_wide"),
    ("c_g8_t6", 1, 8, 4, 3, 6, 4, 2, 0.02, "normal"),        # eight v-heads per k-head
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_chunk_matches_oracle(case):
    name, Hk, Hv, W, B, T, P, steps, std, gates = case
    wl = wl_of(name, Hk, Hv, W, B, T, P, steps, std=std, gate_mode=gates)
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


def test_chunk_is_deterministic():
    wl = wl_of("c_det", 4, 8, 4, 12, 16, 12, 1)
    outs = []
    for _ in range(2):
        g = DeviceRun(wl)
        out, out32 = g.step(g.inputs(0))
        torch.cuda.synchronize()
        outs.append((out32.clone(), g.state.clone(), g.conv.clone()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_chunk_under_graph_replay_with_device_batch():
    # one graph captured at B_max = 6 serves batch counts 6, 2, 0, 5 (sequences 0..B-1)
    wl = wl_of("c_graph", 2, 4, 4, 6, 4, 8, 4)
    g = DeviceRun(wl)
    o = OracleRun(wl, list(range(wl.batch)))
    x_buf = g.inputs(0)
    shape = (wl.batch, wl.tokens, wl.num_v_heads, wl.head_v_dim)
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(shape, dtype=torch.float32, device="cuda")
    bdev = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call():
        gdn.gdn_decode_step_device_batch(g.cfg, bdev, x_buf["qkv"], x_buf["a"], x_buf["b"], x_buf["z"], g.conv_w,
                                         g.A_log, g.dt_bias, g.norm_w, g.conv, g.state, g.slots, out, out32, g.err,
                                         g.workspace)
    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=side):
        call()
    torch.cuda.synchronize()
    import oracle
    for step, B in enumerate([6, 2, 0, 5]):
        x = g.inputs(step)
        for k in x_buf:
            x_buf[k].copy_(x[k])
        bdev.fill_(B)
        out32.fill_(-7.0)
        graph.replay()
        torch.cuda.synchronize()
        assert int(g.err.item()) == 0
        if B > 0:
            xo = synth.step_inputs(wl, step, rows=list(range(B)))
            w = o.w
            r = oracle.decode_step(o.shape, xo["qkv"], xo["a"], xo["b"], xo["z"], w["conv_w"], w["A_log"],
                                   w["dt_bias"], w["norm_w"], o.conv, o.state, o.local[:B])
            compare_out(out[:B], out32[:B], r["out"], list(range(B)), f"graph step {step} B={B}")
        assert torch.all(out32[B:] == -7.0)
    compare_state(g.state, o.state, o.slot_ids, "c_graph")
    np.testing.assert_array_equal(bf16_host(g.conv)[o.slot_ids], o.conv)
    del graph

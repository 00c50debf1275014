"""GPU: one CUDA graph of gdn_decode_step_device_batch, captured once at B_max,
serves every batch count up to B_max. Each replay processes the sequences 0..B-1
named by the device batch count; the oracle advances exactly those sequences at that
step. Bars as for the decode step (outputs within 2e-3, states within 1e-4 per slot
and head, conv history bit-exact); the sequences past the count keep their pools and
their output rows bit-identical."""
import numpy as np
import pytest
import torch

import gated_delta_rule_102_b200 as gdn
import oracle
from gated_delta_rule_102_b200 import synth
from gdn_harness import DeviceRun, OracleRun, bf16_host, compare_out, compare_state

pytestmark = pytest.mark.gpu

SENTINEL = -7.0


def replay_batches(wl, batches):
    g = DeviceRun(wl)
    o = OracleRun(wl, list(range(wl.batch)))
    B_max, T = wl.batch, wl.tokens
    shape = (B_max, T, wl.num_v_heads, wl.head_v_dim)
    x_buf = g.inputs(0)                    # the captured input buffers (refilled before each replay)
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(shape, dtype=torch.float32, device="cuda")
    bdev = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call():
        gdn.gdn_decode_step_device_batch(g.cfg, bdev, x_buf["qkv"], x_buf["a"], x_buf["b"], x_buf["z"], g.conv_w,
                                         g.A_log, g.dt_bias, g.norm_w, g.conv, g.state, g.slots, out, out32, g.err,
                                         g.workspace)
    call()  # the first call, with a count of 0, sets up the host side and changes nothing
    torch.cuda.synchronize()
    state0, conv0 = g.state.clone(), g.conv.clone()
    assert torch.equal(g.state, state0) and int(g.err.item()) == 0
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=side):
        call()
    torch.cuda.synchronize()
    for step, B in enumerate(batches):
        x = g.inputs(step)
        for k in x_buf:
            x_buf[k].copy_(x[k])
        bdev.fill_(B)
        out32.fill_(SENTINEL)
        out.fill_(SENTINEL)
        before_state, before_conv = g.state.clone(), g.conv.clone()
        graph.replay()
        torch.cuda.synchronize()
        assert int(g.err.item()) == 0
        if B > 0:
            xo = synth.step_inputs(wl, step, rows=list(range(B)))
            w = o.w
            r = oracle.decode_step(o.shape, xo["qkv"], xo["a"], xo["b"], xo["z"], w["conv_w"], w["A_log"],
                                   w["dt_bias"], w["norm_w"], o.conv, o.state, o.local[:B])
            compare_out(out[:B], out32[:B], r["out"], list(range(B)), f"{wl.name} step {step} B={B}")
        assert torch.all(out32[B:] == SENTINEL) and torch.all(out[B:].float() == SENTINEL)
        rest = torch.tensor(g.slots_np[B:].tolist(), dtype=torch.long, device="cuda")
        if rest.numel():
            assert torch.equal(g.state[rest], before_state[rest]) and torch.equal(g.conv[rest], before_conv[rest])
    compare_state(g.state, o.state, o.slot_ids, wl.name)
    np.testing.assert_array_equal(bf16_host(g.conv)[o.slot_ids], o.conv)
    # a count outside [0, B_max] runs nothing and is flagged
    bdev.fill_(B_max + 1)
    before = g.state.clone()
    graph.replay()
    torch.cuda.synchronize()
    assert int(g.err.item()) == gdn.GDN_DEVICE_ERR_BATCH and torch.equal(g.state, before)
    del graph


def test_graph_at_batch64_serves_smaller_batches():
    # the persistent single-token kernel (B_max = 64 of the batch64 shape)
    replay_batches(synth.WORKLOADS["batch64"].replace(steps=5), [64, 37, 1, 0, 64])


def test_graph_small_batch_cluster_kernel():
    wl = synth.WORKLOADS["tiny_d16"].replace(name="graph_small", batch=3, pool_slots=5, slot_mode="sample", seed=91)
    replay_batches(wl, [3, 2, 0, 1, 3])


def test_graph_multitoken_kernel():
    wl = synth.WORKLOADS["tiny_d16"].replace(name="graph_mt", num_k_heads=2, num_v_heads=4, head_k_dim=64,
                                             head_v_dim=64, batch=5, tokens=4, pool_slots=7, slot_mode="sample",
                                             state_std=0.02, seed=92)
    replay_batches(wl, [5, 3, 0, 5])

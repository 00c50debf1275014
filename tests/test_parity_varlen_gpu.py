"""gdn_decode_step_varlen: sequences with their own token counts (0 to T_max) packed
row after row in one launch, against the oracle run per sequence with its own count
(the ragged launch is defined as each sequence's tokens processed in order)."""
import zlib

import numpy as np
import pytest
import torch

import gated_delta_rule_102_b200 as gdn
import oracle
from gated_delta_rule_102_b200 import synth
from gdn_harness import OUT_ABS_TOL, DeviceRun, OracleRun, bf16_dev, bf16_host, compare_state

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["tiny_d16"]

VARLEN = [
    # name                Hk Hv   dk   dv  W   B   P  T_max steps
    ("varlen_d128", 2, 4, 128, 128, 4, 6, 8, 16, 3),
    ("varlen_g8_dv64_w3", 1, 8, 64, 64, 3, 5, 6, 7, 2),
    ("varlen_b40", 4, 8, 128, 128, 4, 40, 44, 5, 2),
    ("varlen_dk16_w8", 2, 4, 16, 32, 8, 4, 4, 9, 3),
]


def wl_of(name, Hk, Hv, dk, dv, W, B, P):
    return BASE.replace(name=name, num_k_heads=Hk, num_v_heads=Hv, head_k_dim=dk, head_v_dim=dv, conv_width=W,
                        batch=B, tokens=1, pool_slots=P, seed=zlib.crc32(name.encode()) % 10000, slot_mode="sample",
                        state_std=0.02)


def launch(g, wl, cu_np, t_max, x, want_f32=True):
    total = int(cu_np[-1])
    cu = torch.from_numpy(cu_np.astype(np.int32)).cuda()
    xd = {k: bf16_dev(v) for k, v in x.items()}
    out = torch.empty((total, wl.num_v_heads, wl.head_v_dim), dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(out.shape, dtype=torch.float32, device="cuda") if want_f32 else None
    gdn.gdn_decode_step_varlen(g.cfg, cu, t_max, xd["qkv"], xd["a"], xd["b"], xd["z"], g.conv_w, g.A_log, g.dt_bias,
                               g.norm_w, g.conv, g.state, g.slots, out, out32, g.err)
    return out, out32


def check_rows(out, out32, ref, what):
    g32 = out32.cpu().numpy().astype(np.float64)
    err = np.abs(g32 - ref).max() if ref.size else 0.0
    assert err <= OUT_ABS_TOL, f"{what}: out max abs err {err:.3e}"
    assert np.array_equal(bf16_host(out), synth.to_bf16_bits(out32.cpu().numpy())), what


@pytest.mark.parametrize("spec", VARLEN, ids=[v[0] for v in VARLEN])
def test_varlen_matches_oracle(spec):
    name, Hk, Hv, dk, dv, W, B, P, t_max, steps = spec
    wl = wl_of(name, Hk, Hv, dk, dv, W, B, P)
    g = DeviceRun(wl)
    rows = sorted({0, 1, 2, B // 2, B - 1})
    o = OracleRun(wl, rows)
    pool0 = g.state.clone()
    for s in range(steps):
        counts = synth.varlen_counts(wl, s, t_max)
        cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
        out, out32 = launch(g, wl, cu, t_max, synth.varlen_inputs(wl, s, counts))
        for j, r in enumerate(rows):
            n = int(counts[r])
            if n == 0:
                continue
            x = synth.varlen_inputs(wl, s, counts, rows=[r])
            res = oracle.decode_step(o.shape, x["qkv"][None], x["a"][None], x["b"][None], x["z"][None], o.w["conv_w"],
                                     o.w["A_log"], o.w["dt_bias"], o.w["norm_w"], o.conv, o.state,
                                     np.array([j], dtype=np.int32))
            lo, hi = int(cu[r]), int(cu[r + 1])
            check_rows(out[lo:hi], out32[lo:hi], res["out"][0], f"{name} step {s} sequence {r} ({n} tokens)")
    torch.cuda.synchronize()
    assert int(g.err.item()) == 0
    compare_state(g.state, o.state, o.slot_ids, name)
    np.testing.assert_array_equal(bf16_host(g.conv)[o.slot_ids], o.conv)
    idle = sorted(set(range(P)) - set(g.slots_np.tolist()))
    if idle:
        idx = torch.tensor(idle, device="cuda")
        assert torch.equal(g.state[idx], pool0[idx])


def test_varlen_bad_counts_are_skipped_and_flagged():
    wl = wl_of("varlen_bad", 2, 4, 64, 64, 4, 5, 6)
    g = DeviceRun(wl)
    state0, conv0 = g.state.clone(), g.conv.clone()
    t_max = 4
    counts = np.array([2, 6, 3, 1, 2], dtype=np.int64)       # sequence 1 brings more than t_max
    cu = np.concatenate([[0], np.cumsum(counts)])
    x = synth.varlen_inputs(wl, 0, counts)
    out, out32 = launch(g, wl, cu, t_max, x)
    torch.cuda.synchronize()
    assert int(g.err.item()) & gdn.GDN_DEVICE_ERR_SEQLEN
    s1 = int(g.slots_np[1])
    assert torch.equal(g.state[s1], state0[s1]) and torch.equal(g.conv[s1], conv0[s1])
    # the others went ahead
    for r in (0, 2, 3, 4):
        s = int(g.slots_np[r])
        assert not torch.equal(g.state[s], state0[s])


def test_varlen_rows_past_the_end_are_skipped_and_flagged():
    wl = wl_of("varlen_past_end", 2, 4, 64, 64, 4, 3, 4)
    g = DeviceRun(wl)
    state0 = g.state.clone()
    counts = np.array([2, 3, 1], dtype=np.int64)
    x = synth.varlen_inputs(wl, 0, counts)
    cu = np.array([0, 2, 5, 7])                              # the last sequence claims row 6 of 6 rows
    x = {k: v[:6] for k, v in x.items()}
    total = 6
    cu_d = torch.from_numpy(cu.astype(np.int32)).cuda()
    xd = {k: bf16_dev(v) for k, v in x.items()}
    out = torch.empty((total, 4, 64), dtype=torch.bfloat16, device="cuda")
    gdn.gdn_decode_step_varlen(g.cfg, cu_d, 4, xd["qkv"], xd["a"], xd["b"], xd["z"], g.conv_w, g.A_log, g.dt_bias,
                               g.norm_w, g.conv, g.state, g.slots, out, None, g.err)
    torch.cuda.synchronize()
    assert int(g.err.item()) & gdn.GDN_DEVICE_ERR_SEQLEN
    s2 = int(g.slots_np[2])
    assert torch.equal(g.state[s2], state0[s2])


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_equals_uniform_launch(d):
    # every sequence with T tokens: the ragged entry point gives the uniform one's bits (both
    # take the register kernel at d = 64 and the chunked tensor-core kernel at d = 128)
    wl = wl_of(f"varlen_uniform_d{d}", 2, 4, d, d, 4, 4, 6).replace(tokens=5)
    a, b = DeviceRun(wl), DeviceRun(wl)
    x = a.inputs(0)
    out_u, out_u32 = a.step(x)
    B, T = wl.batch, wl.tokens
    cu = np.arange(B + 1) * T
    flat = {k: bf16_host(v).reshape((B * T,) + tuple(v.shape[2:])) for k, v in x.items()}
    out_v, out_v32 = launch(b, wl, cu, T, flat)
    torch.cuda.synchronize()
    assert torch.equal(a.conv, b.conv)
    assert torch.equal(out_u32.reshape(out_v32.shape), out_v32)
    assert torch.equal(a.state, b.state)

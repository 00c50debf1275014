"""GPU parity of the fused decode step (gdn_decode_step through the C ABI) against
the FP64 oracle, on the five synthetic workloads at full size.

Bars: conv pool and slot indexing bit-exact; fp32 output within 2e-3 absolute of
the oracle (bf16 output within one bf16 ulp of the oracle's correctly rounded
value); state per (slot, head) within 1e-4 of the oracle relative to the head's
largest entry. Full-size workloads compare a sample of sequences with the oracle
one by one (sequences are independent) and check the whole conv pool and every
idle slot exactly."""
import numpy as np
import pytest
import torch

from gated_delta_rule_102_b200 import synth
from gdn_harness import (OUT_ABS_GUARD, STATE_REL_GUARD, DeviceRun, OracleRun, bf16_host, compare_out, compare_state,
                         conv_pool_reference)

pytestmark = pytest.mark.gpu


def _run(wl, rows, check_every=1, state_guard=STATE_REL_GUARD):
    g = DeviceRun(wl)
    o = OracleRun(wl, rows)
    pool0 = g.state.clone() if wl.pool_slots > wl.batch else None
    worst_out = 0.0
    for s in range(wl.steps):
        out, out32 = g.step(g.inputs(s))
        r = o.step(s)
        if s % check_every == 0 or s == wl.steps - 1:
            worst_out = max(worst_out, compare_out(out, out32, r["out"], rows, f"{wl.name} step {s}"))
    torch.cuda.synchronize()
    assert int(g.err.item()) == 0
    worst_state = compare_state(g.state, o.state, o.slot_ids, wl.name)
    # the conv history of EVERY slot, bit for bit
    np.testing.assert_array_equal(bf16_host(g.conv), conv_pool_reference(wl, wl.steps))
    if pool0 is not None:  # slots no sequence names keep their bytes
        idle = sorted(set(range(wl.pool_slots)) - set(g.slots_np.tolist()))
        idx = torch.tensor(idle, device="cuda")
        assert torch.equal(g.state[idx], pool0[idx])
    # far inside the bars: where these kernels' errors actually are
    assert worst_out <= OUT_ABS_GUARD, f"{wl.name}: out error {worst_out:.3e} above the precision guard"
    if state_guard is not None:
        assert worst_state <= state_guard, f"{wl.name}: state error {worst_state:.3e} above the precision guard"
    return worst_out, worst_state


def test_tiny_d16_8_steps():
    wl = synth.WORKLOADS["tiny_d16"]
    _run(wl, rows=[0])


def test_single_sequence_256_steps():
    wl = synth.WORKLOADS["single_seq"]
    _run(wl, rows=[0], state_guard=None)  # (256 steps of rounding in the state: the bar alone)


def test_batch64_64_steps_every_sequence():
    wl = synth.WORKLOADS["batch64"]
    _run(wl, rows=list(range(wl.batch)), check_every=4)


def test_pool384_batch256_32_steps_every_sequence():
    wl = synth.WORKLOADS["pool384_batch256"]
    _run(wl, rows=list(range(wl.batch)), check_every=4)


def test_multitoken_b32_t16_16_launches_every_sequence():
    wl = synth.WORKLOADS["multitoken_b32_t16"]
    _run(wl, rows=list(range(wl.batch)), check_every=2)

"""GPU: the bounded waits give up and report instead of hanging. A self-test kernel
waits on a barrier phase that nothing completes (no copy in flight, the wait bounded by
the SM cycle counter); it must set GDN_DEVICE_ERR_TIMEOUT after about the requested
number of cycles, and the context must stay usable (a decode step afterwards still
matches the oracle)."""
import pytest
import torch

import gated_delta_rule_102_b200 as gdn
from gated_delta_rule_102_b200 import synth
from gdn_harness import DeviceRun, OracleRun, compare_out, compare_state

pytestmark = pytest.mark.gpu


def test_wait_that_nothing_completes_times_out_and_the_context_survives():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cycles = torch.zeros(1, dtype=torch.int64, device="cuda")
    limit = 4_000_000  # about 2 ms at 2 GHz
    gdn.gdn_selftest_wait_timeout(limit, err, cycles)
    torch.cuda.synchronize()
    assert int(err.item()) == gdn.GDN_DEVICE_ERR_TIMEOUT
    took = int(cycles.item())
    assert limit < took < limit + 10_000_000, took  # gave up soon after the limit, not before
    # the context is usable: a decode step still runs and matches the oracle
    wl = synth.WORKLOADS["tiny_d16"]
    g, o = DeviceRun(wl), OracleRun(wl, [0])
    out, out32 = g.step(g.inputs(0))
    r = o.step(0)
    torch.cuda.synchronize()
    assert int(g.err.item()) == 0
    compare_out(out, out32, r["out"], [0], "after the self-test")
    compare_state(g.state, o.state, o.slot_ids, "after the self-test")

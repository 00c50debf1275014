"""gdn_decode_step_static_scratch: the decode step for callers that cannot allocate
device memory (code inside a host framework that owns the allocator, plugins with a
fixed memory budget, paths that must not call cudaMalloc because it can synchronize
the device). It uses a fixed scratch array the library keeps in device memory in
place of the caller's workspace, and must give what gdn_decode_step gives.

This file is collected last, so a run that stops at the first failure has already
run every other test; it also passes on its own in a fresh process."""
import pytest
import torch

import gated_delta_rule_102_b200 as gdn
from gated_delta_rule_102_b200 import synth
from gdn_harness import DeviceRun

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    # batch64 shape: the single-token kernel that uses the scratch runs here
    wl = synth.WORKLOADS["batch64"].replace(steps=2)
    assert gdn.decode_static_scratch_bytes() >= gdn.decode_workspace_bytes()
    ref = DeviceRun(wl, dynamic=True)     # gdn_decode_step with a caller-allocated workspace
    nal = DeviceRun(wl, dynamic=False)    # same weights, pools and slots; no workspace at all
    shape = (wl.batch, wl.tokens, wl.num_v_heads, wl.head_v_dim)
    for step in range(2):
        x = ref.inputs(step)
        out_r, out_r32 = ref.step(x)
        out_n = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        out_n32 = torch.empty(shape, dtype=torch.float32, device="cuda")
        gdn.gdn_decode_step_static_scratch(nal.cfg, x["qkv"], x["a"], x["b"], x["z"], nal.conv_w, nal.A_log,
                                           nal.dt_bias, nal.norm_w, nal.conv, nal.state, nal.slots, out_n, out_n32,
                                           nal.err)
        torch.cuda.synchronize()
        assert int(nal.err.item()) == 0 and int(ref.err.item()) == 0
        # Both calls run the same dynamically scheduled kernel, and every (sequence, head)
        # is computed by one cluster in a fixed order, so the results are the same bits.
        assert torch.equal(out_n32, out_r32)
        assert torch.equal(out_n, out_r)
        assert torch.equal(nal.state, ref.state)
        assert torch.equal(nal.conv, ref.conv)

"""GPU parity of the projections (gdn_in_proj, gdn_out_proj through the C ABI: the
tcgen05 GEMM) against the oracle's FP64 products.

Tolerance, derived from the arithmetic: a product of two bf16 values is exact in
fp32 (8-bit significands), so the only error is the fp32 summation over K terms, in
whatever order the tensor cores and the split-K reduction take. Any order errs by at
most gamma_(K-1) * sum_k |x_k w_k| with gamma_n = n u / (1 - n u), u = 2^-24; the
test allows twice that (2 K u sum |x w|) for the tensor core's internal rounding.
The bf16 outputs must be exactly the round-to-nearest-even of the fp32 outputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_102_b200 as gdn
import oracle
from gated_delta_rule_102_b200 import synth
from gdn_harness import bf16_dev, bf16_host, cfg_of

pytestmark = pytest.mark.gpu


def bound(x_bits, w_bits):
    K = x_bits.shape[1]
    ax, aw = np.abs(oracle.bf16_to_f64(x_bits)), np.abs(oracle.bf16_to_f64(w_bits))
    return 2.0 * K * 2.0 ** -24 * (ax @ aw.T) + 1e-30


def check(name, gpu32, gpu_bf16_parts, ref, tol):
    g = gpu32.cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    assert np.all(err <= tol), f"{name}: max err {err.max():.3e}, worst err/bound {(err / tol).max():.3f}"
    g16 = np.concatenate([bf16_host(t).reshape(g.shape[0], -1) for t in gpu_bf16_parts], axis=1)
    assert np.array_equal(g16, synth.to_bf16_bits(gpu32.cpu().numpy())), f"{name}: bf16 is not the RNE of fp32"
    return float((err / tol).max())


def run_in_proj(wl, rows, hidden, step=0, seed_w=None):
    w = synth.proj_weights(wl if seed_w is None else wl.replace(seed=seed_w), hidden)
    x = synth.proj_inputs(wl, step, rows, hidden)["x"]
    cfg = cfg_of(wl)
    C, Z, Hv = wl.channels, wl.num_v_heads * wl.head_v_dim, wl.num_v_heads
    dev = lambda n: torch.empty(rows, n, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    qkv, z, a, b = dev(C), dev(Z), dev(Hv), dev(Hv)
    out32 = torch.empty(rows, C + Z + 2 * Hv, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.gdn_in_proj(cfg, bf16_dev(x), bf16_dev(w["w_in"]), qkv, z, a, b, out32, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle.in_proj(oracle.Shape.of(wl), x, w["w_in"])
    return check(f"in_proj {wl.name} rows={rows} hidden={hidden}", out32, (qkv, z, a, b), ref["all"],
                 bound(x, w["w_in"])), (qkv, z, a, b, out32)


def run_out_proj(wl, rows, hidden, step=0):
    w = synth.proj_weights(wl, hidden)
    y = synth.proj_inputs(wl, step, rows, hidden)["y"]
    cfg = cfg_of(wl)
    out = torch.empty(rows, hidden, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(rows, hidden, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.gdn_out_proj(cfg, bf16_dev(y), bf16_dev(w["w_out"]), out, out32, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle.out_proj(oracle.Shape.of(wl), y, w["w_out"])
    return check(f"out_proj {wl.name} rows={rows} hidden={hidden}", out32, (out,), ref, bound(y, w["w_out"]))


def test_in_and_out_proj_batch64_hidden2048():
    # the batch64 decode shape (Hk=16, Hv=32, d=128: 12352 stacked in_proj rows) at hidden 2048
    wl = synth.WORKLOADS["batch64"]
    run_in_proj(wl, 64, synth.HIDDEN)
    run_out_proj(wl, 64, synth.HIDDEN)


BASE = synth.WORKLOADS["tiny_d16"]
SHAPES = [
    # name          Hk Hv  dk  dv  rows hidden
    ("tiny_r1", 2, 2, 16, 16, 1, 64),
    ("tiny_r5_h136", 2, 2, 16, 16, 5, 136),      # K not a multiple of 64: a ragged last block
    ("g2_r17_h520", 2, 4, 32, 64, 17, 520),
    ("d128_r100", 4, 8, 128, 128, 100, 1024),
    ("d128_r256", 16, 32, 128, 128, 256, 2048),  # the most rows one call takes
    ("d64_r33_h8", 1, 2, 64, 16, 33, 8),         # hidden = 8: one partial K block
]


@pytest.mark.parametrize("spec", SHAPES, ids=[s[0] for s in SHAPES])
def test_proj_shapes(spec):
    name, Hk, Hv, dk, dv, rows, hidden = spec
    wl = BASE.replace(name=name, num_k_heads=Hk, num_v_heads=Hv, head_k_dim=dk, head_v_dim=dv, seed=77)
    run_in_proj(wl, rows, hidden)
    run_out_proj(wl, rows, hidden)


def test_proj_is_deterministic_and_rejects_oversize():
    wl = BASE.replace(name="det", num_k_heads=2, num_v_heads=4, head_k_dim=32, head_v_dim=32, seed=5)
    _, first = run_in_proj(wl, 24, 256)
    _, second = run_in_proj(wl, 24, 256)
    for t1, t2 in zip(first, second):
        assert torch.equal(t1, t2)
    cfg = cfg_of(wl)
    x = torch.zeros(257, 256, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(wl.channels + 4 * 32 + 8, 256, dtype=torch.bfloat16, device="cuda")
    o = lambda n: torch.zeros(257, n, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    with pytest.raises(gdn.GdnError):
        gdn.gdn_in_proj(cfg, x, w, o(wl.channels), o(128), o(4), o(4))


def test_first_call_in_a_fresh_process_with_a_short_k():
    # K below four 64-element blocks skips the occupancy query; the kernel's shared-memory
    # limit must still be raised before the first launch of the process
    import os
    import subprocess
    import sys
    code = (
        "import sys, torch; sys.path.insert(0, 'tests'); import gated_delta_rule_102_b200 as gdn\n"
        "from gated_delta_rule_102_b200 import synth\n"
        "from gdn_harness import cfg_of\n"
        "wl = synth.WORKLOADS['tiny_d16'].replace(num_k_heads=1, num_v_heads=2, head_k_dim=64, head_v_dim=16)\n"
        "cfg = cfg_of(wl); rows, hidden = 33, 8\n"
        "x = torch.randn(rows, hidden, device='cuda').to(torch.bfloat16)\n"
        "w = torch.randn(wl.channels + 2 * 16 + 4, hidden, device='cuda').to(torch.bfloat16)\n"
        "o = lambda n: torch.empty(rows, n, dtype=torch.bfloat16, device='cuda')\n"
        "gdn.gdn_in_proj(cfg, x, w, o(wl.channels), o(32), o(2), o(2)); torch.cuda.synchronize(); print('ok')\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stderr[-2000:]

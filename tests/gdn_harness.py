"""Shared machinery of the GPU parity tests: one synthetic workload run through the
CUDA path (C ABI, device pools) and, for a chosen subset of its sequences, through
the FP64 oracle (host pools). Both sides get the same generated bits."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import gated_delta_rule_102_b200 as gdn
import oracle
from gated_delta_rule_102_b200 import synth

# Tolerances (the derivation is in the design notes):
OUT_ABS_TOL = 2e-3        # fp32 output vs oracle, O(1) outputs
STATE_REL_TOL = 1e-4      # per (slot, head): max|dS| / max|S_ref|
# Guards ten and five times inside those bars, where the fused fp32 kernels' errors sit ~100x
# lower (1e-6 outputs, 1e-7..1e-6 states in short runs): a change that gives away an order of
# magnitude of precision fails here long before it nears the bars.
OUT_ABS_GUARD = 2e-4
STATE_REL_GUARD = 2e-5


def bf16_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(device).view(torch.bfloat16)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def f32_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def cfg_of(wl: synth.Workload) -> gdn.GdnConfig:
    return gdn.GdnConfig.make(wl.num_k_heads, wl.num_v_heads, wl.head_k_dim, wl.head_v_dim, wl.conv_width)


class DeviceRun:
    """The workload on the GPU: weights, pools and slots resident on the device."""

    def __init__(self, wl: synth.Workload, device="cuda", state0: Optional[np.ndarray] = None,
                 dynamic: bool = True):
        self.wl, self.device = wl, device
        self.workspace = gdn.decode_workspace(device) if dynamic else None
        self.cfg = cfg_of(wl)
        w = synth.weights(wl)
        self.conv_w = bf16_dev(w["conv_w"], device)
        self.A_log = f32_dev(w["A_log"], device)
        self.dt_bias = f32_dev(w["dt_bias"], device)
        self.norm_w = bf16_dev(w["norm_w"], device)
        self.slots_np = synth.slots(wl)
        self.slots = torch.from_numpy(self.slots_np).to(device)
        s0 = synth.initial_state(wl) if state0 is None else state0
        self.state = f32_dev(s0, device)
        self.conv = bf16_dev(synth.initial_conv_state(wl), device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)

    def inputs(self, step: int) -> Dict[str, torch.Tensor]:
        x = synth.step_inputs(self.wl, step)
        return {k: bf16_dev(v, self.device) for k, v in x.items()}

    def step(self, x: Dict[str, torch.Tensor], want_f32=True):
        wl = self.wl
        shape = (wl.batch, wl.tokens, wl.num_v_heads, wl.head_v_dim)
        out = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        out32 = torch.empty(shape, dtype=torch.float32, device=self.device) if want_f32 else None
        gdn.gdn_decode_step(self.cfg, x["qkv"], x["a"], x["b"], x["z"], self.conv_w, self.A_log, self.dt_bias,
                            self.norm_w, self.conv, self.state, self.slots, out, out32, self.err, self.workspace)
        return out, out32


class OracleRun:
    """The same workload in the FP64 oracle, for the sequences `rows` only (each
    sequence is independent, so a subset reproduces its part of the full run)."""

    def __init__(self, wl: synth.Workload, rows: Sequence[int], state0: Optional[np.ndarray] = None):
        self.wl, self.rows = wl, list(rows)
        self.shape = oracle.Shape.of(wl)
        self.w = synth.weights(wl)
        slots = synth.slots(wl)
        self.slot_ids = [int(slots[r]) for r in self.rows]
        s0 = synth.initial_state(wl, self.slot_ids) if state0 is None else state0[self.slot_ids]
        self.state = s0.astype(np.float64)
        self.conv = synth.initial_conv_state(wl, self.slot_ids)
        self.local = np.arange(len(self.rows), dtype=np.int32)

    def step(self, step: int) -> Dict[str, np.ndarray]:
        x = synth.step_inputs(self.wl, step, rows=self.rows)
        w = self.w
        n = len(self.rows)
        if n < 8:
            return oracle.decode_step(self.shape, x["qkv"], x["a"], x["b"], x["z"], w["conv_w"], w["A_log"],
                                      w["dt_bias"], w["norm_w"], self.conv, self.state, self.local)
        # Sequences are independent: contiguous shards of rows run in threads (the oracle's C
        # calls release the interpreter lock), each on its own slice of the pools.
        nth = min(n // 4, os.cpu_count() or 1, 32)
        cuts = [n * i // nth for i in range(nth + 1)]

        def shard(i):
            a, b = cuts[i], cuts[i + 1]
            return oracle.decode_step(self.shape, x["qkv"][a:b], x["a"][a:b], x["b"][a:b], x["z"][a:b],
                                      w["conv_w"], w["A_log"], w["dt_bias"], w["norm_w"], self.conv[a:b],
                                      self.state[a:b], np.arange(b - a, dtype=np.int32))
        with ThreadPoolExecutor(max_workers=nth) as ex:
            parts = list(ex.map(shard, range(nth)))
        return {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}


def conv_pool_reference(wl: synth.Workload, steps: int) -> np.ndarray:
    """Conv history of every slot after `steps` launches, from the oracle's conv stage
    (cheap: no state), for the bit-exact check of the whole pool."""
    sh = oracle.Shape.of(wl)
    pool = synth.initial_conv_state(wl)
    slots = synth.slots(wl)
    w = synth.weights(wl)
    for s in range(steps):
        x = synth.step_inputs(wl, s)
        oracle.conv_update(sh, x["qkv"], w["conv_w"], pool, slots)
    return pool


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def compare_out(gpu_bf16: torch.Tensor, gpu_f32: torch.Tensor, ref: np.ndarray, rows: List[int], what=""):
    """fp32 output within OUT_ABS_TOL of the oracle, and the bf16 output exactly the
    round-to-nearest-even of that fp32 value (so |bf16 - oracle| <= tol + ulp/2).
    A per-element relative bound would be wrong: outputs near zero come from
    cancellation and carry an absolute, not a relative, error."""
    g32 = gpu_f32.cpu().numpy()[rows]
    err = np.abs(g32.astype(np.float64) - ref)
    assert err.max() <= OUT_ABS_TOL, f"{what}: out max abs err {err.max():.3e}"
    gb = bf16_host(gpu_bf16)[rows]
    mism = gb != synth.to_bf16_bits(g32)
    assert not mism.any(), f"{what}: {mism.sum()} bf16 outputs are not the RNE of the fp32 output"
    gbf = synth.bf16_bits_to_f32(gb).astype(np.float64)
    ulp = bf16_ulp(np.maximum(np.abs(ref), np.abs(g32.astype(np.float64))))
    assert np.all(np.abs(gbf - ref) <= OUT_ABS_TOL + 0.5 * ulp * 1.0000001), what
    return float(err.max())


def compare_state(gpu_state: torch.Tensor, ref_state: np.ndarray, slot_ids: List[int], what=""):
    g = gpu_state[torch.tensor(slot_ids, device=gpu_state.device)].cpu().numpy().astype(np.float64)
    diff = np.abs(g - ref_state).reshape(len(slot_ids), ref_state.shape[1], -1).max(-1)
    scale = np.abs(ref_state).reshape(len(slot_ids), ref_state.shape[1], -1).max(-1)
    rel = diff / np.maximum(scale, 1e-30)
    assert rel.max() <= STATE_REL_TOL, f"{what}: state max rel err {rel.max():.3e}"
    return float(rel.max())

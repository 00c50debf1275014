"""Seeded synthetic inputs for the GDN decode step.

This module is the one thing the CUDA path and the FP64 oracle share. It draws
random numbers and rounds them to the storage types (bf16 bit patterns, fp32);
it computes nothing of the method itself.

Generator
---------
Every tensor is a counter-based stream: value ``i`` of the stream with key
``K`` is ``splitmix64_mix(K + (i + 1) * 0x9E3779B97F4A7C15)``, the output
function of Steele, Lea and Flood's SplitMix64 (OOPSLA 2014). The key hashes
``(seed, tensor name, indices)`` with 64-bit FNV-1a followed by the same mix,
so one step or one pool slot can be regenerated alone (the sampled parity
checks at full size rely on that).

* uniform in [0, 1): the top 53 bits of a draw times 2**-53;
* normal: Box-Muller on consecutive draw pairs (u1, u2):
  ``r = sqrt(-2 ln(1 - u1))``, values ``r cos(2 pi u2)`` then ``r sin(2 pi u2)``;
* bf16: the float64 draw is rounded to float32 (round-to-nearest-even), then
  the float32 to bf16 (round-to-nearest-even on the top 16 bits).

"N(0, s)" everywhere means standard deviation ``s``.

Workloads
---------
``WORKLOADS`` holds the five synthetic decode workloads (shapes, batch, pool,
steps, distributions) that the tests and the benchmark use.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional, Sequence

import numpy as np

_GOLDEN = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1


def _mix_int(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, name: str, *idx: int) -> int:
    """64-bit key of the stream for tensor ``name`` at indices ``idx``."""
    h = 0xCBF29CE484222325
    for byte in f"{seed}|{name}|{'/'.join(str(i) for i in idx)}".encode():
        h = ((h ^ byte) * 0x100000001B3) & _M64
    return _mix_int(h)


def raw_u64(key: int, n: int) -> np.ndarray:
    """The first ``n`` 64-bit outputs of the SplitMix64 stream ``key``."""
    with np.errstate(over="ignore"):
        ctr = np.arange(1, n + 1, dtype=np.uint64) * np.uint64(_GOLDEN)
        return _mix(ctr + np.uint64(key & _M64))


def uniform(key: int, n: int, lo: float = 0.0, hi: float = 1.0) -> np.ndarray:
    u = (raw_u64(key, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return lo + (hi - lo) * u


def normal(key: int, n: int, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    m = (n + 1) // 2
    u = uniform(key, 2 * m)
    r = np.sqrt(-2.0 * np.log1p(-u[0::2]))
    th = 2.0 * math.pi * u[1::2]
    z = np.empty(2 * m, dtype=np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    return mean + std * z[:n]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64/float32 array -> bf16 bit patterns (uint16), both roundings RNE."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact widening)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    ``slot_mode``: ``identity`` (slot b for sequence b), ``permutation`` (a
    seeded permutation of the pool) or ``sample`` (``batch`` distinct slots
    drawn without replacement from a larger pool).
    ``gate_mode``: ``normal`` (a ~ N(0,1) like the other projections) or
    ``decay_half_to_one`` (a chosen so that exp(g) is spread over [0.5, 1)) or
    ``decay_wide`` (exp(g) = 2^-u with u ~ U(0, 48), and 2^-200 for about one entry
    in eight: decays far below 1, down to values that underflow in fp32).
    ``ragged``: each launch gives every sequence its own token count, 0..``tokens``
    (``varlen_counts``), packed row after row (``varlen_inputs``).
    """

    name: str
    num_k_heads: int
    num_v_heads: int
    head_k_dim: int
    head_v_dim: int
    conv_width: int
    batch: int
    tokens: int
    pool_slots: int
    steps: int
    state_std: float
    slot_mode: str
    gate_mode: str
    seed: int
    ragged: bool = False

    @property
    def channels(self) -> int:
        return 2 * self.num_k_heads * self.head_k_dim + self.num_v_heads * self.head_v_dim

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


_QWEN3_NEXT_LIKE = dict(num_k_heads=16, num_v_heads=32, head_k_dim=128, head_v_dim=128, conv_width=4)

WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in (
        Workload("tiny_d16", num_k_heads=2, num_v_heads=2, head_k_dim=16, head_v_dim=16, conv_width=4,
                 batch=1, tokens=1, pool_slots=1, steps=8, state_std=0.0, slot_mode="identity",
                 gate_mode="normal", seed=1000),
        Workload("single_seq", **_QWEN3_NEXT_LIKE, batch=1, tokens=1, pool_slots=1, steps=256,
                 state_std=0.02, slot_mode="identity", gate_mode="normal", seed=1001),
        Workload("batch64", **_QWEN3_NEXT_LIKE, batch=64, tokens=1, pool_slots=64, steps=64,
                 state_std=0.02, slot_mode="permutation", gate_mode="normal", seed=1002),
        Workload("pool384_batch256", **_QWEN3_NEXT_LIKE, batch=256, tokens=1, pool_slots=384, steps=32,
                 state_std=0.02, slot_mode="sample", gate_mode="decay_half_to_one", seed=1003),
        Workload("multitoken_b32_t16", **_QWEN3_NEXT_LIKE, batch=32, tokens=16, pool_slots=32, steps=16,
                 state_std=0.02, slot_mode="permutation", gate_mode="normal", seed=1004),
        Workload("ragged_b64_t16", **_QWEN3_NEXT_LIKE, batch=64, tokens=16, pool_slots=64, steps=8,
                 state_std=0.02, slot_mode="permutation", gate_mode="normal", seed=1005, ragged=True),
    )
}


def weights(wl: Workload) -> Dict[str, np.ndarray]:
    """Layer parameters: conv_w [C][W] bf16 ~ N(0,0.5); A_log [Hv] fp32 ~ U(-1,1);
    dt_bias [Hv] fp32 ~ N(0,0.1); norm_w [dv] bf16 ~ 1 + N(0,0.05)."""
    C, W, Hv, dv = wl.channels, wl.conv_width, wl.num_v_heads, wl.head_v_dim
    return {
        "conv_w": to_bf16_bits(normal(stream_key(wl.seed, "conv_w"), C * W, 0.5)).reshape(C, W),
        "A_log": uniform(stream_key(wl.seed, "A_log"), Hv, -1.0, 1.0).astype(np.float32),
        "dt_bias": normal(stream_key(wl.seed, "dt_bias"), Hv, 0.1).astype(np.float32),
        "norm_w": to_bf16_bits(normal(stream_key(wl.seed, "norm_w"), dv, 0.05, 1.0)),
    }


def slots(wl: Workload) -> np.ndarray:
    """int32 [B]: the pool slot of each sequence."""
    if wl.slot_mode == "identity":
        return np.arange(wl.batch, dtype=np.int32)
    order = np.argsort(uniform(stream_key(wl.seed, "slots"), wl.pool_slots), kind="stable")
    if wl.slot_mode == "permutation":
        assert wl.batch == wl.pool_slots
    return order[: wl.batch].astype(np.int32)


def _seq_rows(wl: Workload, rows: Optional[Sequence[int]]) -> Iterable[int]:
    return range(wl.batch) if rows is None else rows


def step_inputs(wl: Workload, step: int, rows: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    """Per-step projections for the sequences ``rows`` (default: all), each drawn
    from its own (step, sequence) stream so a subset regenerates identically.

    qkv [n][T][C], a [n][T][Hv], b [n][T][Hv], z [n][T][Hv][dv]: bf16 bits.
    """
    T, C, Hv, dv = wl.tokens, wl.channels, wl.num_v_heads, wl.head_v_dim
    rows = list(_seq_rows(wl, rows))
    out = {k: [] for k in ("qkv", "a", "b", "z")}
    w = weights(wl) if wl.gate_mode != "normal" else None
    for r in rows:
        out["qkv"].append(normal(stream_key(wl.seed, "qkv", step, r), T * C))
        out["b"].append(normal(stream_key(wl.seed, "b", step, r), T * Hv))
        out["z"].append(normal(stream_key(wl.seed, "z", step, r), T * Hv * dv))
        if wl.gate_mode == "normal":
            out["a"].append(normal(stream_key(wl.seed, "a", step, r), T * Hv))
        else:
            # Choose the decay d = exp(g) and invert the gate's parameterisation for
            # the raw projection a (input construction only): -ln d = exp(A_log)
            # softplus(a + dt_bias).
            if wl.gate_mode == "decay_half_to_one":
                neg_ln_d = -np.log(uniform(stream_key(wl.seed, "decay", step, r), T * Hv, 0.5, 1.0 - 2.0 ** -8))
            else:
                u = uniform(stream_key(wl.seed, "decay", step, r), T * Hv, 0.0, 48.0)
                tiny = uniform(stream_key(wl.seed, "decay_tiny", step, r), T * Hv, 0.0, 1.0) < 0.125
                neg_ln_d = np.where(tiny, 200.0, u) * np.log(2.0)
            A = np.tile(w["A_log"].astype(np.float64), T)
            y = neg_ln_d / np.exp(A)
            out["a"].append(np.log(np.expm1(y)) - np.tile(w["dt_bias"].astype(np.float64), T))
    n = len(rows)
    return {
        "qkv": to_bf16_bits(np.concatenate(out["qkv"]) if n else np.zeros(0)).reshape(n, T, C),
        "a": to_bf16_bits(np.concatenate(out["a"]) if n else np.zeros(0)).reshape(n, T, Hv),
        "b": to_bf16_bits(np.concatenate(out["b"]) if n else np.zeros(0)).reshape(n, T, Hv),
        "z": to_bf16_bits(np.concatenate(out["z"]) if n else np.zeros(0)).reshape(n, T, Hv, dv),
    }


def varlen_counts(wl: Workload, step: int, t_max: int) -> np.ndarray:
    """int32 [B]: token counts of a ragged launch, each in 0..t_max: sequence 0 gets
    t_max, sequence 1 one token, sequence 2 none (when the batch has them), the rest
    uniform draws."""
    u = uniform(stream_key(wl.seed, "varlen", step), wl.batch)
    n = np.minimum((u * (t_max + 1)).astype(np.int64), t_max)
    for i, v in enumerate((t_max, 1, 0)[: wl.batch]):
        n[i] = v
    return n.astype(np.int32)


def varlen_inputs(wl: Workload, step: int, counts: Sequence[int],
                  rows: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    """Inputs of a ragged launch packed row after row (the sequences `rows`, default
    all, in order; sequence i brings counts[i] tokens): qkv [total][C], a, b
    [total][Hv], z [total][Hv][dv]. Sequence i's tokens are the first counts[i]
    tokens of its own (step, sequence) streams, so a subset regenerates alone."""
    C, Hv, dv = wl.channels, wl.num_v_heads, wl.head_v_dim
    rows = list(_seq_rows(wl, rows))
    parts = {k: [] for k in ("qkv", "a", "b", "z")}
    for r in rows:
        n = int(counts[r])
        if n <= 0:
            continue
        x = step_inputs(wl.replace(tokens=n), step, rows=[r])
        for k in parts:
            parts[k].append(x[k][0])
    shapes = {"qkv": (C,), "a": (Hv,), "b": (Hv,), "z": (Hv, dv)}
    return {k: (np.concatenate(v) if v else np.zeros((0,) + shapes[k], dtype=np.uint16)) for k, v in parts.items()}


def initial_state(wl: Workload, slot_ids: Optional[Sequence[int]] = None) -> np.ndarray:
    """fp32 [n][Hv][dk][dv]: initial delta-rule state of the given pool slots
    (default: every slot), N(0, state_std) per slot stream, or zeros."""
    slot_ids = range(wl.pool_slots) if slot_ids is None else slot_ids
    per = wl.num_v_heads * wl.head_k_dim * wl.head_v_dim
    ids = list(slot_ids)
    out = np.zeros((len(ids), wl.num_v_heads, wl.head_k_dim, wl.head_v_dim), dtype=np.float32)
    if wl.state_std > 0:
        for i, s in enumerate(ids):
            out[i] = normal(stream_key(wl.seed, "S0", s), per, wl.state_std).reshape(out.shape[1:])
    return out


def initial_conv_state(wl: Workload, slot_ids: Optional[Sequence[int]] = None) -> np.ndarray:
    """bf16 bits [n][W-1][C]: the conv history starts at zeros."""
    n = wl.pool_slots if slot_ids is None else len(list(slot_ids))
    return np.zeros((n, wl.conv_width - 1, wl.channels), dtype=np.uint16)


# Model width of the projections around the layer: a Qwen3-Next-like model with this
# GDN head shape (16 k-heads, 32 v-heads of 128) has hidden size 2048.
HIDDEN = 2048


def proj_weights(wl: Workload, hidden: int = HIDDEN) -> Dict[str, np.ndarray]:
    """Random-initialised projection weights (no trained checkpoint): the stacked
    in_proj w_in [C + Hv*dv + 2*Hv][hidden] (rows: qkv | z | a | b) and out_proj w_out
    [hidden][Hv*dv], bf16 bits ~ N(0, 0.02)."""
    C, Z, Hv = wl.channels, wl.num_v_heads * wl.head_v_dim, wl.num_v_heads
    n_in = C + Z + 2 * Hv
    return {
        "w_in": to_bf16_bits(normal(stream_key(wl.seed, "w_in"), n_in * hidden, 0.02)).reshape(n_in, hidden),
        "w_out": to_bf16_bits(normal(stream_key(wl.seed, "w_out"), hidden * Z, 0.02)).reshape(hidden, Z),
    }


def proj_inputs(wl: Workload, step: int, rows: int, hidden: int = HIDDEN) -> Dict[str, np.ndarray]:
    """Per-step inputs of the projections for `rows` token rows: the normalised layer
    input x [rows][hidden] and the gated decode output y [rows][Hv*dv], bf16 bits ~ N(0, 1)."""
    Z = wl.num_v_heads * wl.head_v_dim
    return {
        "x": to_bf16_bits(normal(stream_key(wl.seed, "x_norm", step), rows * hidden)).reshape(rows, hidden),
        "y": to_bf16_bits(normal(stream_key(wl.seed, "y_gated", step), rows * Z)).reshape(rows, Z),
    }

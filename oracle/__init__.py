"""FP64 CPU oracle for the GDN decode step (ctypes wrapper over ``gdn_oracle.c``).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the CUDA product path
never does. It shares no code with the CUDA path: the one common input is the
seeded generator in ``gated_delta_rule_102_b200.synth``, which draws numbers and
holds none of the method's arithmetic.

Source: the page "spark_model/forward/qwen3_5/linear_attention.rs", steps 3-8 and
the SiLU(z) gate of steps 9+10+11, with the gated delta rule of step 7. The C
file's header states every layout.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("num_k_heads", ctypes.c_int), ("num_v_heads", ctypes.c_int),
                ("head_k_dim", ctypes.c_int), ("head_v_dim", ctypes.c_int),
                ("conv_width", ctypes.c_int), ("l2_eps", ctypes.c_double),
                ("rms_eps", ctypes.c_double), ("q_scale", ctypes.c_double)]


@dataclass(frozen=True)
class Shape:
    num_k_heads: int
    num_v_heads: int
    head_k_dim: int
    head_v_dim: int
    conv_width: int
    l2_eps: float = 1e-6
    rms_eps: float = 1e-6
    q_scale: float = 0.0

    @property
    def channels(self) -> int:
        return 2 * self.num_k_heads * self.head_k_dim + self.num_v_heads * self.head_v_dim

    def _c(self) -> _Cfg:
        return _Cfg(self.num_k_heads, self.num_v_heads, self.head_k_dim, self.head_v_dim,
                    self.conv_width, self.l2_eps, self.rms_eps, self.q_scale)

    @staticmethod
    def of(wl) -> "Shape":
        return Shape(wl.num_k_heads, wl.num_v_heads, wl.head_k_dim, wl.head_v_dim, wl.conv_width)


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i = ctypes.c_void_p, ctypes.c_int
        cp = ctypes.POINTER(_Cfg)
        lib.oracle_conv_update.argtypes = [cp, i, i, vp, vp, vp, i, vp, vp, vp, vp]
        lib.oracle_gate.argtypes = [cp, i, vp, vp, vp, vp, vp, vp]
        lib.oracle_delta_rule.argtypes = [cp, i, i, vp, vp, vp, vp, vp, vp, i, vp, vp]
        lib.oracle_delta_rule_matrix_form.argtypes = [cp, i, i, vp, vp, vp, vp, vp, vp, i, vp, vp]
        lib.oracle_gated_rmsnorm.argtypes = [cp, i, vp, vp, vp, vp]
        lib.oracle_decode_step.argtypes = [cp, i, i] + [vp] * 10 + [i, vp] + [vp] * 7
        lib.oracle_round_bf16.argtypes = [vp, vp, ctypes.c_size_t]
        for f in ("oracle_conv_update", "oracle_gate", "oracle_delta_rule",
                  "oracle_delta_rule_matrix_form", "oracle_gated_rmsnorm", "oracle_decode_step",
                  "oracle_round_bf16"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray], dtype):
    if a is None:
        return None
    assert a.dtype == dtype and a.flags.c_contiguous, (a.dtype, dtype)
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def conv_update(shape: Shape, qkv, conv_w, conv_pool: np.ndarray, slots):
    """Step 3 (+ q scale). ``conv_pool`` (uint16 [P][W-1][C]) is rolled in place.
    Returns q, k [B][T][Hk][dk] and v [B][T][Hv][dv] as float64."""
    lib = _load()
    qkv, conv_w, slots = _u16(qkv), _u16(conv_w), _i32(slots)
    B, T, C = qkv.shape
    assert C == shape.channels and conv_pool.dtype == np.uint16 and conv_pool.flags.c_contiguous
    q = np.zeros((B, T, shape.num_k_heads, shape.head_k_dim))
    k = np.zeros_like(q)
    v = np.zeros((B, T, shape.num_v_heads, shape.head_v_dim))
    lib.oracle_conv_update(ctypes.byref(shape._c()), B, T, _p(qkv, np.uint16), _p(conv_w, np.uint16),
                           _p(conv_pool, np.uint16), conv_pool.shape[0], _p(slots, np.int32),
                           _p(q, np.float64), _p(k, np.float64), _p(v, np.float64))
    return q, k, v


def gate(shape: Shape, a, b, A_log, dt_bias):
    """Steps 4-5. Returns (alpha = exp(g), beta) with a's shape [..., Hv], float64."""
    lib = _load()
    a, b = _u16(a), _u16(b)
    rows = a.size // shape.num_v_heads
    alpha = np.zeros(a.shape)
    beta = np.zeros(a.shape)
    lib.oracle_gate(ctypes.byref(shape._c()), rows, _p(a, np.uint16), _p(b, np.uint16),
                    _p(_f32(A_log), np.float32), _p(_f32(dt_bias), np.float32),
                    _p(alpha, np.float64), _p(beta, np.float64))
    return alpha, beta


def _delta(fn, shape: Shape, q, k, v, alpha, beta, state_pool: np.ndarray, slots):
    lib = _load()
    q, k, v, alpha, beta, slots = _f64(q), _f64(k), _f64(v), _f64(alpha), _f64(beta), _i32(slots)
    B, T = q.shape[:2]
    assert state_pool.dtype == np.float64 and state_pool.flags.c_contiguous
    o = np.zeros((B, T, shape.num_v_heads, shape.head_v_dim))
    getattr(lib, fn)(ctypes.byref(shape._c()), B, T, _p(q, np.float64), _p(k, np.float64),
                     _p(v, np.float64), _p(alpha, np.float64), _p(beta, np.float64),
                     _p(state_pool, np.float64), state_pool.shape[0], _p(slots, np.int32),
                     _p(o, np.float64))
    return o


def delta_rule(shape: Shape, q, k, v, alpha, beta, state_pool: np.ndarray, slots):
    """Step 7 in the stated order; ``state_pool`` (float64 [P][Hv][dk][dv]) is
    updated in place. Returns o [B][T][Hv][dv]."""
    return _delta("oracle_delta_rule", shape, q, k, v, alpha, beta, state_pool, slots)


def delta_rule_matrix_form(shape: Shape, q, k, v, alpha, beta, state_pool: np.ndarray, slots):
    """Step 7 as S' = alpha (I - beta k k^T) S + beta k v^T (cross-check only)."""
    return _delta("oracle_delta_rule_matrix_form", shape, q, k, v, alpha, beta, state_pool, slots)


def gated_rmsnorm(shape: Shape, o, z, norm_w):
    """Step 8 + SiLU(z) gate. ``o`` float [..., dv], ``z`` bf16 bits of the same shape."""
    lib = _load()
    o, z = _f64(o), _u16(z)
    out = np.zeros(o.shape)
    lib.oracle_gated_rmsnorm(ctypes.byref(shape._c()), o.size // shape.head_v_dim, _p(o, np.float64),
                             _p(z, np.uint16), _p(_u16(norm_w), np.uint16), _p(out, np.float64))
    return out


def decode_step(shape: Shape, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w,
                conv_pool: np.ndarray, state_pool: np.ndarray, slots) -> Dict[str, np.ndarray]:
    """One decode launch (all stages). Pools are updated in place. Returns the
    output and every intermediate as float64 arrays."""
    lib = _load()
    qkv, a, b, z, slots = _u16(qkv), _u16(a), _u16(b), _u16(z), _i32(slots)
    B, T = qkv.shape[:2]
    Hk, Hv, dk, dv = shape.num_k_heads, shape.num_v_heads, shape.head_k_dim, shape.head_v_dim
    assert conv_pool.dtype == np.uint16 and conv_pool.flags.c_contiguous
    assert state_pool.dtype == np.float64 and state_pool.flags.c_contiguous
    r = {"out": np.zeros((B, T, Hv, dv)), "q": np.zeros((B, T, Hk, dk)), "k": np.zeros((B, T, Hk, dk)),
         "v": np.zeros((B, T, Hv, dv)), "alpha": np.zeros((B, T, Hv)), "beta": np.zeros((B, T, Hv)),
         "o": np.zeros((B, T, Hv, dv))}
    lib.oracle_decode_step(ctypes.byref(shape._c()), B, T, _p(qkv, np.uint16), _p(a, np.uint16),
                           _p(b, np.uint16), _p(z, np.uint16), _p(_u16(conv_w), np.uint16),
                           _p(_f32(A_log), np.float32), _p(_f32(dt_bias), np.float32),
                           _p(_u16(norm_w), np.uint16), _p(conv_pool, np.uint16),
                           _p(state_pool, np.float64), state_pool.shape[0], _p(slots, np.int32),
                           _p(r["out"], np.float64), _p(r["q"], np.float64), _p(r["k"], np.float64),
                           _p(r["v"], np.float64), _p(r["alpha"], np.float64), _p(r["beta"], np.float64),
                           _p(r["o"], np.float64))
    return r


def round_bf16(x) -> np.ndarray:
    """Correctly rounded (RNE) bf16 bit patterns of float64 values."""
    lib = _load()
    x = _f64(x)
    out = np.zeros(x.shape, dtype=np.uint16)
    lib.oracle_round_bf16(_p(x, np.float64), _p(out, np.uint16), ctypes.c_size_t(x.size))
    return out


def speculative_step(shape: Shape, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w,
                     conv_pool: np.ndarray, state_pool: np.ndarray, slots, n_accept) -> Dict[str, np.ndarray]:
    """Speculative decoding of T drafted tokens with rollback to the accepted prefix,
    written out from its definition: the returned outputs are those of a T-token
    decode step (every drafted token is scored), and the pools end as after a decode
    step over only the first n_accept[b] tokens of each sequence b. The GDN
    counterpart of rewinding a rejected draft ("metrale_model_arch/glm5next_dsa/layer.rs",
    the lockstep check and rewind_to): the recurrent state cannot be truncated, so
    the accepted prefix is what the pools must hold.

    Pools are updated in place (sequences are independent, so each is advanced on its
    own); n_accept[b] = 0 leaves sequence b's pool entries untouched."""
    qkv, a, b, z, slots = _u16(qkv), _u16(a), _u16(b), _u16(z), _i32(slots)
    B, T = qkv.shape[:2]
    n_accept = np.asarray(n_accept, dtype=np.int64)
    assert n_accept.shape == (B,) and np.all((n_accept >= 0) & (n_accept <= T))
    # every drafted token scored, on copies of the pools
    r = decode_step(shape, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool.copy(), state_pool.copy(), slots)
    for i in range(B):
        n = int(n_accept[i])
        if n == 0:
            continue
        decode_step(shape, qkv[i:i + 1, :n], a[i:i + 1, :n], b[i:i + 1, :n], z[i:i + 1, :n], conv_w, A_log,
                    dt_bias, norm_w, conv_pool, state_pool, slots[i:i + 1])
    return r


def bf16_to_f64(bits) -> np.ndarray:
    """The exact values of bf16 bit patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def linear(x_bits, w_bits) -> np.ndarray:
    """out[r][n] = sum_k x[r][k] w[n][k] in FP64 on the exact bf16 values (a library
    matmul as the one step: the products are exact, the sums FP64). The form of every
    projection GEMV on the page "spark_model/forward/qwen3_5/linear_attention.rs"
    (x @ W^T with W stored as [out_features][in_features])."""
    x, w = bf16_to_f64(x_bits), bf16_to_f64(w_bits)
    assert x.ndim == 2 and w.ndim == 2 and x.shape[1] == w.shape[1]
    return x @ w.T


def in_proj(shape: Shape, x_bits, w_in_bits) -> Dict[str, np.ndarray]:
    """Step 2 of the page: the projections of the normalised input x_norm [R][hidden]
    into qkv [R][C], z [R][Hv*dv] and the gate and beta inputs a, b [R][Hv], with the
    four weights stacked row-wise in that order: w_in [C + Hv*dv + 2*Hv][hidden]
    (in_proj_qkv | in_proj_z | in_proj_a | in_proj_b)."""
    y = linear(x_bits, w_in_bits)
    C, Z, Hv = shape.channels, shape.num_v_heads * shape.head_v_dim, shape.num_v_heads
    assert y.shape[1] == C + Z + 2 * Hv
    return {"qkv": y[:, :C], "z": y[:, C:C + Z], "a": y[:, C + Z:C + Z + Hv], "b": y[:, C + Z + Hv:], "all": y}


def out_proj(shape: Shape, y_bits, w_out_bits) -> np.ndarray:
    """The GEMV of the page's fused steps 9+10+11: out = out_proj @ y with y [R][Hv*dv]
    the SiLU(z)-gated, normalised decode output and w_out [hidden][Hv*dv]."""
    assert np.asarray(y_bits).shape[1] == shape.num_v_heads * shape.head_v_dim
    return linear(y_bits, w_out_bits)

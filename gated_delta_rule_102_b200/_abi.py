"""ctypes binding of libgdn (include/gdn.h): the same entry points, argument
marshalling only. Tensors are torch CUDA tensors (bf16 arguments as
torch.bfloat16, whose storage is the bf16 bit pattern); the call goes to the
caller's current CUDA stream unless ``stream`` is given.

There is no fallback: if libgdn.so is missing or cannot be loaded, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK = 0
GDN_ERR_INVALID_ARGUMENT = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_MISALIGNED = 3
GDN_ERR_SLOT_RANGE = 4
GDN_ERR_CUDA = 5
GDN_DEVICE_ERR_SLOT_RANGE = 1
GDN_DEVICE_ERR_TIMEOUT = 2
GDN_DEVICE_ERR_SEQLEN = 4
GDN_DEVICE_ERR_BATCH = 8

EXPORTS = ("gdn_conv_update", "gdn_recurrent_step", "gdn_gated_rmsnorm", "gdn_decode_step",
           "gdn_decode_workspace_bytes", "gdn_decode_step_varlen", "gdn_decode_step_static_scratch",
           "gdn_decode_static_scratch_bytes", "gdn_spec_verify", "gdn_spec_commit", "gdn_in_proj", "gdn_out_proj",
           "gdn_decode_step_device_batch", "gdn_selftest_wait_timeout",
           "gdn_check_slots_host", "gdn_status_string", "gdn_abi_version")


class GdnConfig(ctypes.Structure):
    """Mirror of ``gdn_config``."""
    _fields_ = [("num_k_heads", ctypes.c_int32), ("num_v_heads", ctypes.c_int32),
                ("head_k_dim", ctypes.c_int32), ("head_v_dim", ctypes.c_int32),
                ("conv_width", ctypes.c_int32), ("l2_eps", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("q_scale", ctypes.c_float)]

    @classmethod
    def make(cls, num_k_heads, num_v_heads, head_k_dim, head_v_dim, conv_width,
             l2_eps=1e-6, rms_eps=1e-6, q_scale=0.0) -> "GdnConfig":
        return cls(num_k_heads, num_v_heads, head_k_dim, head_v_dim, conv_width, l2_eps, rms_eps, q_scale)

    @property
    def channels(self) -> int:
        return 2 * self.num_k_heads * self.head_k_dim + self.num_v_heads * self.head_v_dim


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libgdn with argument types declared (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libgdn.so not built at {LIB_PATH}; run python -m gated_delta_rule_102_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32 = ctypes.c_void_p, ctypes.c_int32
        cfgp = ctypes.POINTER(GdnConfig)
        L.gdn_conv_update.argtypes = [cfgp, i32, i32, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp]
        L.gdn_recurrent_step.argtypes = [cfgp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp]
        L.gdn_gated_rmsnorm.argtypes = [cfgp, i32, vp, vp, vp, vp, vp, vp]
        L.gdn_decode_step.argtypes = [cfgp, i32, i32] + [vp] * 10 + [i32, vp, vp, vp, vp, vp, vp]
        L.gdn_decode_step_varlen.argtypes = [cfgp, i32, vp, i32, i32] + [vp] * 10 + [i32, vp, vp, vp, vp, vp]
        L.gdn_decode_workspace_bytes.argtypes = []
        L.gdn_decode_workspace_bytes.restype = ctypes.c_size_t
        L.gdn_decode_step_static_scratch.argtypes = [cfgp, i32, i32] + [vp] * 10 + [i32, vp, vp, vp, vp, vp]
        L.gdn_decode_step_static_scratch.restype = ctypes.c_int32
        L.gdn_decode_static_scratch_bytes.argtypes = []
        L.gdn_decode_static_scratch_bytes.restype = ctypes.c_size_t
        L.gdn_spec_verify.argtypes = [cfgp, i32, i32] + [vp] * 10 + [i32] + [vp] * 8
        L.gdn_spec_commit.argtypes = [cfgp, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp]
        L.gdn_decode_step_device_batch.argtypes = [cfgp, vp, i32, i32] + [vp] * 10 + [i32, vp, vp, vp, vp, vp, vp]
        L.gdn_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp, vp, vp]
        L.gdn_selftest_wait_timeout.restype = ctypes.c_int32
        L.gdn_in_proj.argtypes = [cfgp, i32, i32] + [vp] * 9
        L.gdn_out_proj.argtypes = [cfgp, i32, i32] + [vp] * 6
        L.gdn_check_slots_host.argtypes = [vp, i32, i32]
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_abi_version.argtypes = []
        for f in ("gdn_conv_update", "gdn_recurrent_step", "gdn_gated_rmsnorm", "gdn_decode_step",
                  "gdn_decode_step_varlen", "gdn_spec_verify", "gdn_spec_commit", "gdn_in_proj", "gdn_out_proj",
                  "gdn_decode_step_device_batch", "gdn_check_slots_host",
                  "gdn_abi_version"):
            getattr(L, f).restype = ctypes.c_int32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != GDN_OK:
        raise GdnError(status, where)


def _ptr(t: Optional[torch.Tensor], dtypes, name: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)
_F32 = (torch.float32,)
_I32 = (torch.int32,)
_WS = (torch.int32, torch.uint8, torch.int64)


def _stream(stream, ref: torch.Tensor):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(ref.device).cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def gdn_conv_update(cfg: GdnConfig, qkv, conv_w, conv_pool, slots, q_out, k_out, v_out,
                    err_flag=None, stream=None) -> None:
    B, T = qkv.shape[0], qkv.shape[1]
    _check(lib().gdn_conv_update(ctypes.byref(cfg), B, T, _ptr(qkv, _BF16, "qkv"), _ptr(conv_w, _BF16, "conv_w"),
                                 _ptr(conv_pool, _BF16, "conv_pool"), conv_pool.shape[0],
                                 _ptr(slots, _I32, "slots"), _ptr(q_out, _F32, "q_out"),
                                 _ptr(k_out, _F32, "k_out"), _ptr(v_out, _F32, "v_out"),
                                 _ptr(err_flag, _I32, "err_flag"), _stream(stream, qkv)), "gdn_conv_update")


def gdn_recurrent_step(cfg: GdnConfig, q, k, v, a, b, A_log, dt_bias, state_pool, slots, o,
                       err_flag=None, stream=None) -> None:
    B, T = q.shape[0], q.shape[1]
    _check(lib().gdn_recurrent_step(ctypes.byref(cfg), B, T, _ptr(q, _F32, "q"), _ptr(k, _F32, "k"),
                                    _ptr(v, _F32, "v"), _ptr(a, _BF16, "a"), _ptr(b, _BF16, "b"),
                                    _ptr(A_log, _F32, "A_log"), _ptr(dt_bias, _F32, "dt_bias"),
                                    _ptr(state_pool, _F32, "state_pool"), state_pool.shape[0],
                                    _ptr(slots, _I32, "slots"), _ptr(o, _F32, "o"),
                                    _ptr(err_flag, _I32, "err_flag"), _stream(stream, q)), "gdn_recurrent_step")


def gdn_gated_rmsnorm(cfg: GdnConfig, o, z, norm_w, out, out_f32=None, stream=None) -> None:
    rows = o.numel() // cfg.head_v_dim
    _check(lib().gdn_gated_rmsnorm(ctypes.byref(cfg), rows, _ptr(o, _F32, "o"), _ptr(z, _BF16, "z"),
                                   _ptr(norm_w, _BF16, "norm_w"), _ptr(out, _BF16, "out"),
                                   _ptr(out_f32, _F32, "out_f32"), _stream(stream, o)), "gdn_gated_rmsnorm")


def gdn_decode_step(cfg: GdnConfig, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool,
                    slots, out, out_f32=None, err_flag=None, workspace=None, stream=None) -> None:
    B, T = qkv.shape[0], qkv.shape[1]
    _check(lib().gdn_decode_step(ctypes.byref(cfg), B, T, _ptr(qkv, _BF16, "qkv"), _ptr(a, _BF16, "a"),
                                 _ptr(b, _BF16, "b"), _ptr(z, _BF16, "z"), _ptr(conv_w, _BF16, "conv_w"),
                                 _ptr(A_log, _F32, "A_log"), _ptr(dt_bias, _F32, "dt_bias"),
                                 _ptr(norm_w, _BF16, "norm_w"), _ptr(conv_pool, _BF16, "conv_pool"),
                                 _ptr(state_pool, _F32, "state_pool"), state_pool.shape[0],
                                 _ptr(slots, _I32, "slots"), _ptr(out, _BF16, "out"),
                                 _ptr(out_f32, _F32, "out_f32"), _ptr(err_flag, _I32, "err_flag"),
                                 _ptr(workspace, _WS, "workspace"), _stream(stream, qkv)), "gdn_decode_step")


def gdn_decode_step_device_batch(cfg: GdnConfig, B_dev, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool,
                                 state_pool, slots, out, out_f32=None, err_flag=None, workspace=None,
                                 stream=None) -> None:
    """gdn_decode_step sized for B_max = qkv.shape[0] sequences that runs the first
    B_dev[0] of them (B_dev: a one-element int32 CUDA tensor read on the device), so a
    captured CUDA graph serves any batch up to B_max."""
    B, T = qkv.shape[0], qkv.shape[1]
    _check(lib().gdn_decode_step_device_batch(
        ctypes.byref(cfg), _ptr(B_dev, _I32, "B_dev"), B, T, _ptr(qkv, _BF16, "qkv"), _ptr(a, _BF16, "a"),
        _ptr(b, _BF16, "b"), _ptr(z, _BF16, "z"), _ptr(conv_w, _BF16, "conv_w"), _ptr(A_log, _F32, "A_log"),
        _ptr(dt_bias, _F32, "dt_bias"), _ptr(norm_w, _BF16, "norm_w"), _ptr(conv_pool, _BF16, "conv_pool"),
        _ptr(state_pool, _F32, "state_pool"), state_pool.shape[0], _ptr(slots, _I32, "slots"), _ptr(out, _BF16, "out"),
        _ptr(out_f32, _F32, "out_f32"), _ptr(err_flag, _I32, "err_flag"), _ptr(workspace, _WS, "workspace"),
        _stream(stream, qkv)), "gdn_decode_step_device_batch")


def gdn_decode_step_varlen(cfg: GdnConfig, cu_seqlens, T_max: int, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w,
                           conv_pool, state_pool, slots, out, out_f32=None, err_flag=None, stream=None) -> None:
    """The decode step for sequences with their own token counts, packed row after row:
    sequence i owns rows cu_seqlens[i] .. cu_seqlens[i+1]-1 of qkv [total][C], a, b
    [total][Hv], z and out [total][Hv][dv]; T_max bounds every count."""
    B = cu_seqlens.shape[0] - 1
    total = qkv.shape[0]
    _check(lib().gdn_decode_step_varlen(
        ctypes.byref(cfg), B, _ptr(cu_seqlens, _I32, "cu_seqlens"), int(T_max), total, _ptr(qkv, _BF16, "qkv"),
        _ptr(a, _BF16, "a"), _ptr(b, _BF16, "b"), _ptr(z, _BF16, "z"), _ptr(conv_w, _BF16, "conv_w"),
        _ptr(A_log, _F32, "A_log"), _ptr(dt_bias, _F32, "dt_bias"), _ptr(norm_w, _BF16, "norm_w"),
        _ptr(conv_pool, _BF16, "conv_pool"), _ptr(state_pool, _F32, "state_pool"), state_pool.shape[0],
        _ptr(slots, _I32, "slots"), _ptr(out, _BF16, "out"), _ptr(out_f32, _F32, "out_f32"),
        _ptr(err_flag, _I32, "err_flag"), _stream(stream, qkv)), "gdn_decode_step_varlen")


def gdn_decode_step_static_scratch(cfg: GdnConfig, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool,
                                   state_pool, slots, out, out_f32=None, err_flag=None, stream=None) -> None:
    """gdn_decode_step for callers that cannot allocate: the library's own fixed device
    scratch replaces the workspace (calls that overlap on the GPU race on it)."""
    B, T = qkv.shape[0], qkv.shape[1]
    _check(lib().gdn_decode_step_static_scratch(
        ctypes.byref(cfg), B, T, _ptr(qkv, _BF16, "qkv"), _ptr(a, _BF16, "a"), _ptr(b, _BF16, "b"),
        _ptr(z, _BF16, "z"), _ptr(conv_w, _BF16, "conv_w"), _ptr(A_log, _F32, "A_log"),
        _ptr(dt_bias, _F32, "dt_bias"), _ptr(norm_w, _BF16, "norm_w"), _ptr(conv_pool, _BF16, "conv_pool"),
        _ptr(state_pool, _F32, "state_pool"), state_pool.shape[0], _ptr(slots, _I32, "slots"),
        _ptr(out, _BF16, "out"), _ptr(out_f32, _F32, "out_f32"), _ptr(err_flag, _I32, "err_flag"),
        _stream(stream, qkv)), "gdn_decode_step_static_scratch")


def gdn_spec_verify(cfg: GdnConfig, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool, slots,
                    out, spec_k, spec_delta, spec_alpha, out_f32=None, err_flag=None, stream=None) -> None:
    """Verify T drafted tokens (qkv [B][T][C], ...): the outputs of a T-token decode step,
    the pools untouched, and per token the normalised key spec_k [B][T][Hk][dk], the
    write spec_delta [B][T][Hv][dv] and the decay spec_alpha [B][T][Hv] (fp32)."""
    B, T = qkv.shape[0], qkv.shape[1]
    _check(lib().gdn_spec_verify(
        ctypes.byref(cfg), B, T, _ptr(qkv, _BF16, "qkv"), _ptr(a, _BF16, "a"), _ptr(b, _BF16, "b"),
        _ptr(z, _BF16, "z"), _ptr(conv_w, _BF16, "conv_w"), _ptr(A_log, _F32, "A_log"),
        _ptr(dt_bias, _F32, "dt_bias"), _ptr(norm_w, _BF16, "norm_w"), _ptr(conv_pool, _BF16, "conv_pool"),
        _ptr(state_pool, _F32, "state_pool"), state_pool.shape[0], _ptr(slots, _I32, "slots"),
        _ptr(out, _BF16, "out"), _ptr(out_f32, _F32, "out_f32"), _ptr(spec_k, _F32, "spec_k"),
        _ptr(spec_delta, _F32, "spec_delta"), _ptr(spec_alpha, _F32, "spec_alpha"),
        _ptr(err_flag, _I32, "err_flag"), _stream(stream, qkv)), "gdn_spec_verify")


def gdn_spec_commit(cfg: GdnConfig, n_accept, qkv, conv_pool, state_pool, slots, spec_k, spec_delta, spec_alpha,
                    err_flag=None, stream=None) -> None:
    """Keep the first n_accept[b] verified tokens of every sequence b (device int32 [B])."""
    B, T = qkv.shape[0], qkv.shape[1]
    _check(lib().gdn_spec_commit(
        ctypes.byref(cfg), B, T, _ptr(n_accept, _I32, "n_accept"), _ptr(qkv, _BF16, "qkv"),
        _ptr(conv_pool, _BF16, "conv_pool"), _ptr(state_pool, _F32, "state_pool"), state_pool.shape[0],
        _ptr(slots, _I32, "slots"), _ptr(spec_k, _F32, "spec_k"), _ptr(spec_delta, _F32, "spec_delta"),
        _ptr(spec_alpha, _F32, "spec_alpha"), _ptr(err_flag, _I32, "err_flag"), _stream(stream, qkv)),
        "gdn_spec_commit")


def gdn_in_proj(cfg: GdnConfig, x, w_in, qkv, z, a, b, out_f32=None, err_flag=None, stream=None) -> None:
    """[qkv | z | a | b] = x @ w_in^T: x [rows][hidden], w_in [C + Hv*dv + 2*Hv][hidden] (bf16)."""
    rows, hidden = x.shape[0], x.shape[-1]
    _check(lib().gdn_in_proj(ctypes.byref(cfg), hidden, rows, _ptr(x, _BF16, "x"), _ptr(w_in, _BF16, "w_in"),
                             _ptr(qkv, _BF16, "qkv"), _ptr(z, _BF16, "z"), _ptr(a, _BF16, "a"), _ptr(b, _BF16, "b"),
                             _ptr(out_f32, _F32, "out_f32"), _ptr(err_flag, _I32, "err_flag"), _stream(stream, x)),
           "gdn_in_proj")


def gdn_out_proj(cfg: GdnConfig, y, w_out, out, out_f32=None, err_flag=None, stream=None) -> None:
    """out = y @ w_out^T: y [rows][Hv*dv], w_out [hidden][Hv*dv] (bf16), out [rows][hidden]."""
    rows, hidden = y.shape[0], w_out.shape[0]
    _check(lib().gdn_out_proj(ctypes.byref(cfg), hidden, rows, _ptr(y, _BF16, "y"), _ptr(w_out, _BF16, "w_out"),
                              _ptr(out, _BF16, "out"), _ptr(out_f32, _F32, "out_f32"),
                              _ptr(err_flag, _I32, "err_flag"), _stream(stream, y)), "gdn_out_proj")


def decode_static_scratch_bytes() -> int:
    return int(lib().gdn_decode_static_scratch_bytes())


def decode_workspace_bytes() -> int:
    return int(lib().gdn_decode_workspace_bytes())


def decode_workspace(device) -> torch.Tensor:
    """A zeroed workspace for gdn_decode_step on `device` (keep one per stream)."""
    return torch.zeros(decode_workspace_bytes() // 4, dtype=torch.int32, device=device)


def gdn_selftest_wait_timeout(limit_cycles: int, err_flag, cycles=None, stream=None) -> None:
    """Run the bounded-wait self-test: a wait that nothing completes must give up after
    about limit_cycles SM cycles and set GDN_DEVICE_ERR_TIMEOUT in err_flag."""
    _check(lib().gdn_selftest_wait_timeout(int(limit_cycles), _ptr(err_flag, _I32, "err_flag"),
                                           _ptr(cycles, (torch.int64,), "cycles"), _stream(stream, err_flag)),
           "gdn_selftest_wait_timeout")


def gdn_check_slots_host(slots, pool_slots: int) -> int:
    """Status of the host-side slot check on a CPU int32 array-like."""
    import numpy as np
    s = np.ascontiguousarray(np.asarray(slots, dtype=np.int32))
    return int(lib().gdn_check_slots_host(s.ctypes.data_as(ctypes.c_void_p), s.size, int(pool_slots)))


def abi_version() -> int:
    return int(lib().gdn_abi_version())


class DecodePlan:
    """gdn_decode_step with its arguments marshalled once: ``launch()`` makes the
    same C call with the stored pointers, for loops that replay one set of tensors
    (the tensors must stay alive and in place while the plan is used)."""

    def __init__(self, cfg: GdnConfig, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool,
                 slots, out, out_f32=None, err_flag=None, workspace=None, stream=None):
        self._keep = (cfg, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool, slots, out,
                      out_f32, err_flag, workspace)
        self._fn = lib().gdn_decode_step
        self._args = (ctypes.byref(cfg), qkv.shape[0], qkv.shape[1], _ptr(qkv, _BF16, "qkv"), _ptr(a, _BF16, "a"),
                      _ptr(b, _BF16, "b"), _ptr(z, _BF16, "z"), _ptr(conv_w, _BF16, "conv_w"),
                      _ptr(A_log, _F32, "A_log"), _ptr(dt_bias, _F32, "dt_bias"), _ptr(norm_w, _BF16, "norm_w"),
                      _ptr(conv_pool, _BF16, "conv_pool"), _ptr(state_pool, _F32, "state_pool"),
                      state_pool.shape[0], _ptr(slots, _I32, "slots"), _ptr(out, _BF16, "out"),
                      _ptr(out_f32, _F32, "out_f32"), _ptr(err_flag, _I32, "err_flag"),
                      _ptr(workspace, _WS, "workspace"), _stream(stream, qkv))

    def launch(self) -> None:
        st = self._fn(*self._args)
        if st != GDN_OK:
            raise GdnError(st, "gdn_decode_step")

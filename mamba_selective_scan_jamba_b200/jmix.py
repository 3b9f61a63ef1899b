"""Python binding of libjmix (ctypes; argument marshalling only).

Every name mirrors the C ABI in ``include/jmix.h``.  Tensors may be torch
tensors (their ``data_ptr()`` is passed) or raw integer addresses.  Every
computation runs in libjmix's CUDA kernels; if the library is missing this
module raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from typing import Mapping, Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_build", "libjmix.so")

JM_OK, JM_ERR_INVALID_ARG, JM_ERR_UNSUPPORTED, JM_ERR_CUDA, JM_ERR_TIMEOUT, JM_ERR_WORKSPACE = range(6)
JM_F32, JM_BF16 = 0, 1
STATUS_NAMES = {0: "JM_OK", 1: "JM_ERR_INVALID_ARG", 2: "JM_ERR_UNSUPPORTED", 3: "JM_ERR_CUDA",
                4: "JM_ERR_TIMEOUT", 5: "JM_ERR_WORKSPACE"}

WEIGHT_NAMES = ("conv_w", "conv_b", "xproj_w", "dt_norm_w", "b_norm_w", "c_norm_w", "dtproj_w",
                "dt_bias", "A_log", "D")

EXPORTED = ("jm_mixer_fwd_workspace_size", "jm_mixer_step_workspace_size", "jm_mixer_fwd",
            "jm_mixer_step", "jm_mixer_fwd_host", "jm_poll_error", "jm_last_error",
            "jm_last_launch_count", "jm_last_kernel_name", "jm_set_kernel_events",
            "jm_mixer_step_noalloc", "jm_mixer_fwd_schedule",
            "jm_mixer_fwd_varlen_workspace_size", "jm_mixer_fwd_varlen", "jm_selftest_timeout",
            "jm_layer_fwd_workspace_size", "jm_layer_fwd", "jm_scan_bwd_workspace_size",
            "jm_scan_bwd", "jm_scan_bwd_schedule", "jm_noalloc_poll_error",
            "jm_noalloc_selftest_timeout", "jm_prepared_weights_size", "jm_prepare_weights",
            "jm_mixer_step_indexed")


class jm_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("d_inner", ctypes.c_int64), ("d_state", ctypes.c_int64),
                ("d_conv", ctypes.c_int64), ("dt_rank", ctypes.c_int64),
                ("eps", ctypes.c_float), ("io", ctypes.c_int),
                ("discretization", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class JmixError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None
_vp = ctypes.c_void_p


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libjmix.so (built by ``build.build_libjmix``); raises if it is absent."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise FileNotFoundError(f"libjmix is not built ({p}); run __graft_entry__.build()")
    lib = ctypes.CDLL(p)
    lib.jm_mixer_fwd_workspace_size.restype = ctypes.c_size_t
    lib.jm_mixer_fwd_workspace_size.argtypes = [ctypes.POINTER(jm_dims)]
    lib.jm_mixer_step_workspace_size.restype = ctypes.c_size_t
    lib.jm_mixer_step_workspace_size.argtypes = [ctypes.POINTER(jm_dims)]
    lib.jm_mixer_fwd.restype = ctypes.c_int
    lib.jm_mixer_fwd.argtypes = [ctypes.POINTER(jm_dims)] + [_vp] * 18 + [ctypes.c_size_t, _vp]
    lib.jm_mixer_step.restype = ctypes.c_int
    lib.jm_mixer_step.argtypes = [ctypes.POINTER(jm_dims)] + [_vp] * 16 + [ctypes.c_size_t, _vp]
    lib.jm_mixer_step_noalloc.restype = ctypes.c_int
    lib.jm_mixer_step_noalloc.argtypes = [ctypes.POINTER(jm_dims)] + [_vp] * 15 + [_vp]
    lib.jm_mixer_fwd_host.restype = ctypes.c_int
    lib.jm_mixer_fwd_host.argtypes = [ctypes.POINTER(jm_dims)] + [_vp] * 19 + [ctypes.c_size_t, _vp]
    lib.jm_mixer_fwd_varlen_workspace_size.restype = ctypes.c_size_t
    lib.jm_mixer_fwd_varlen_workspace_size.argtypes = [ctypes.POINTER(jm_dims)]
    lib.jm_mixer_fwd_varlen.restype = ctypes.c_int
    lib.jm_mixer_fwd_varlen.argtypes = ([ctypes.POINTER(jm_dims)] + [_vp] * 19
                                        + [ctypes.c_size_t, _vp])
    lib.jm_layer_fwd_workspace_size.restype = ctypes.c_size_t
    lib.jm_layer_fwd_workspace_size.argtypes = [ctypes.POINTER(jm_dims), ctypes.c_int64]
    lib.jm_layer_fwd.restype = ctypes.c_int
    lib.jm_layer_fwd.argtypes = ([ctypes.POINTER(jm_dims), ctypes.c_int64] + [_vp] * 19
                                 + [ctypes.c_size_t, _vp])
    lib.jm_scan_bwd_workspace_size.restype = ctypes.c_size_t
    lib.jm_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(jm_dims)]
    lib.jm_scan_bwd.restype = ctypes.c_int
    lib.jm_scan_bwd.argtypes = [ctypes.POINTER(jm_dims)] + [_vp] * 16 + [ctypes.c_size_t, _vp]
    lib.jm_selftest_timeout.restype = ctypes.c_int
    lib.jm_selftest_timeout.argtypes = [_vp, ctypes.c_size_t, _vp]
    lib.jm_scan_bwd_schedule.restype = ctypes.c_int
    lib.jm_scan_bwd_schedule.argtypes = [ctypes.POINTER(jm_dims), ctypes.POINTER(ctypes.c_int)]
    lib.jm_mixer_fwd_schedule.restype = ctypes.c_int
    lib.jm_mixer_fwd_schedule.argtypes = [ctypes.POINTER(jm_dims), ctypes.POINTER(ctypes.c_int),
                                          ctypes.POINTER(ctypes.c_int)]
    lib.jm_poll_error.restype = ctypes.c_int
    lib.jm_poll_error.argtypes = [_vp, _vp]
    lib.jm_prepared_weights_size.restype = ctypes.c_size_t
    lib.jm_prepared_weights_size.argtypes = [ctypes.POINTER(jm_dims)]
    lib.jm_prepare_weights.restype = ctypes.c_int
    lib.jm_prepare_weights.argtypes = [ctypes.POINTER(jm_dims), _vp, _vp, _vp, ctypes.c_size_t,
                                       _vp]
    lib.jm_mixer_step_indexed.restype = ctypes.c_int
    lib.jm_mixer_step_indexed.argtypes = ([ctypes.POINTER(jm_dims), _vp, ctypes.c_int64]
                                          + [_vp] * 14 + [_vp, _vp, _vp, ctypes.c_size_t, _vp])
    lib.jm_noalloc_poll_error.restype = ctypes.c_int
    lib.jm_noalloc_poll_error.argtypes = [_vp]
    lib.jm_noalloc_selftest_timeout.restype = ctypes.c_int
    lib.jm_noalloc_selftest_timeout.argtypes = [_vp]
    lib.jm_last_error.restype = ctypes.c_char_p
    lib.jm_last_error.argtypes = []
    lib.jm_last_launch_count.restype = ctypes.c_int
    lib.jm_last_launch_count.argtypes = []
    lib.jm_last_kernel_name.restype = ctypes.c_char_p
    lib.jm_last_kernel_name.argtypes = [ctypes.c_int]
    lib.jm_set_kernel_events.restype = ctypes.c_int
    lib.jm_set_kernel_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
    if path is None:
        _lib = lib
    return lib


JM_DISC_EULER, JM_DISC_ZOH = 0, 1


def dims(batch: int, seqlen: int, d_inner: int, dt_rank: int, io: int = JM_BF16,
         eps: float = 1e-6, d_state: int = 16, d_conv: int = 4, zoh: bool = False) -> jm_dims:
    return jm_dims(batch, seqlen, d_inner, d_state, d_conv, dt_rank, eps, io,
                   JM_DISC_ZOH if zoh else JM_DISC_EULER, 0)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int) -> None:
    if status != JM_OK:
        raise JmixError(status, load().jm_last_error().decode())


def jm_mixer_fwd_workspace_size(d: jm_dims) -> int:
    return load().jm_mixer_fwd_workspace_size(ctypes.byref(d))


def jm_mixer_fwd_schedule(d: jm_dims):
    """(n_parts, two_pass) of the scan schedule jm_mixer_fwd uses for these dims."""
    n, t = ctypes.c_int(0), ctypes.c_int(0)
    _check(load().jm_mixer_fwd_schedule(ctypes.byref(d), ctypes.byref(n), ctypes.byref(t)))
    return n.value, bool(t.value)


def jm_scan_bwd_schedule(d: jm_dims) -> int:
    """Time parts per sequence that jm_scan_bwd uses for these dims."""
    n = ctypes.c_int(0)
    _check(load().jm_scan_bwd_schedule(ctypes.byref(d), ctypes.byref(n)))
    return n.value


def jm_mixer_step_workspace_size(d: jm_dims) -> int:
    return load().jm_mixer_step_workspace_size(ctypes.byref(d))


def _weights(w: Mapping):
    return [_ptr(w[k]) for k in WEIGHT_NAMES]


def jm_mixer_fwd(d: jm_dims, x, z, w: Mapping, y, final_state, workspace, ws_bytes: int,
                 init_conv_state=None, init_ssm_state=None, final_conv_state=None,
                 stream=None, check: bool = True) -> int:
    st = load().jm_mixer_fwd(ctypes.byref(d), _ptr(x), _ptr(z), *_weights(w), _ptr(y),
                             _ptr(final_state), _ptr(init_conv_state), _ptr(init_ssm_state),
                             _ptr(final_conv_state), _ptr(workspace), ws_bytes, _stream(stream))
    if check:
        _check(st)
    return st


def jm_layer_fwd_workspace_size(d: jm_dims, d_model: int) -> int:
    return load().jm_layer_fwd_workspace_size(ctypes.byref(d), d_model)


def jm_layer_fwd(d: jm_dims, d_model: int, hidden, in_proj_w, w: Mapping, out_proj_w, out,
                 final_state, workspace, ws_bytes: int, init_conv_state=None,
                 init_ssm_state=None, final_conv_state=None, stream=None,
                 check: bool = True) -> int:
    """The full Mamba layer: in_proj -> mixer core -> out_proj (see include/jmix.h)."""
    st = load().jm_layer_fwd(ctypes.byref(d), d_model, _ptr(hidden), _ptr(in_proj_w),
                             *_weights(w), _ptr(out_proj_w), _ptr(out), _ptr(final_state),
                             _ptr(init_conv_state), _ptr(init_ssm_state),
                             _ptr(final_conv_state), _ptr(workspace), ws_bytes, _stream(stream))
    if check:
        _check(st)
    return st


def jm_scan_bwd_workspace_size(d: jm_dims) -> int:
    return load().jm_scan_bwd_workspace_size(ctypes.byref(d))


def jm_scan_bwd(d: jm_dims, delta, u, Bm, Cm, A_log, D, h0, gy, g_delta, g_u, g_B, g_C,
                g_A_log, g_D, g_h0, workspace, ws_bytes: int, stream=None,
                check: bool = True) -> int:
    """Backward of the scan core (see include/jmix.h); float32 device tensors."""
    st = load().jm_scan_bwd(ctypes.byref(d), *[_ptr(t) for t in (
        delta, u, Bm, Cm, A_log, D, h0, gy, g_delta, g_u, g_B, g_C, g_A_log, g_D, g_h0,
        workspace)], ws_bytes, _stream(stream))
    if check:
        _check(st)
    return st


def jm_selftest_timeout(workspace, ws_bytes: int, stream=None, check: bool = True) -> int:
    """Launch the bounded wait that is never satisfied (see include/jmix.h)."""
    st = load().jm_selftest_timeout(_ptr(workspace), ws_bytes, _stream(stream))
    if check:
        _check(st)
    return st


def jm_mixer_fwd_varlen_workspace_size(d: jm_dims) -> int:
    return load().jm_mixer_fwd_varlen_workspace_size(ctypes.byref(d))


def jm_mixer_fwd_varlen(d: jm_dims, cu_seqlens, x, z, w: Mapping, y, final_state, workspace,
                        ws_bytes: int, init_conv_state=None, init_ssm_state=None,
                        final_conv_state=None, stream=None, check: bool = True) -> int:
    """Packed batch: d.batch sequences, d.seqlen total tokens; cu_seqlens is a device
    int32 tensor of d.batch + 1 offsets."""
    st = load().jm_mixer_fwd_varlen(ctypes.byref(d), _ptr(cu_seqlens), _ptr(x), _ptr(z),
                                    *_weights(w), _ptr(y), _ptr(final_state),
                                    _ptr(init_conv_state), _ptr(init_ssm_state),
                                    _ptr(final_conv_state), _ptr(workspace), ws_bytes,
                                    _stream(stream))
    if check:
        _check(st)
    return st


def jm_mixer_step(d: jm_dims, x_t, z_t, conv_state, ssm_state, w: Mapping, y_t, workspace,
                  ws_bytes: int, stream=None, check: bool = True) -> int:
    st = load().jm_mixer_step(ctypes.byref(d), _ptr(x_t), _ptr(z_t), _ptr(conv_state),
                              _ptr(ssm_state), *_weights(w), _ptr(y_t), _ptr(workspace), ws_bytes,
                              _stream(stream))
    if check:
        _check(st)
    return st


def jm_prepared_weights_size(d: jm_dims) -> int:
    return load().jm_prepared_weights_size(ctypes.byref(d))


def jm_prepare_weights(d: jm_dims, xproj_w, dtproj_w, prepared, nbytes: int, stream=None,
                       check: bool = True) -> int:
    st = load().jm_prepare_weights(ctypes.byref(d), _ptr(xproj_w), _ptr(dtproj_w), _ptr(prepared),
                                   nbytes, _stream(stream))
    if check:
        _check(st)
    return st


def jm_mixer_step_indexed(d: jm_dims, state_idx, n_slots: int, x_t, z_t, conv_pool, ssm_pool,
                          w: Mapping, prepared, y_t, workspace, ws_bytes: int, stream=None,
                          check: bool = True) -> int:
    """One decode step whose rows use slots state_idx[b] of the state pools."""
    st = load().jm_mixer_step_indexed(ctypes.byref(d), _ptr(state_idx), n_slots, _ptr(x_t),
                                      _ptr(z_t), _ptr(conv_pool), _ptr(ssm_pool), *_weights(w),
                                      _ptr(prepared), _ptr(y_t), _ptr(workspace), ws_bytes,
                                      _stream(stream))
    if check:
        _check(st)
    return st


def jm_mixer_step_noalloc(d: jm_dims, x_t, z_t, conv_state, ssm_state, w: Mapping, y_t,
                          stream=None, check: bool = True) -> int:
    """jm_mixer_step with libjmix's static scratch instead of a caller workspace."""
    st = load().jm_mixer_step_noalloc(ctypes.byref(d), _ptr(x_t), _ptr(z_t), _ptr(conv_state),
                                      _ptr(ssm_state), *_weights(w), _ptr(y_t), _stream(stream))
    if check:
        _check(st)
    return st


def jm_mixer_fwd_host(d: jm_dims, x_host, z_host, y_host, final_state_host, x_dev, z_dev, y_dev,
                      final_state_dev, w: Mapping, workspace, ws_bytes: int, stream=None,
                      check: bool = True) -> int:
    st = load().jm_mixer_fwd_host(ctypes.byref(d), _ptr(x_host), _ptr(z_host), _ptr(y_host),
                                  _ptr(final_state_host), _ptr(x_dev), _ptr(z_dev), _ptr(y_dev),
                                  _ptr(final_state_dev), *_weights(w), _ptr(workspace), ws_bytes,
                                  _stream(stream))
    if check:
        _check(st)
    return st


def jm_poll_error(workspace, stream=None) -> int:
    return load().jm_poll_error(_ptr(workspace), _stream(stream))


def jm_noalloc_poll_error(stream=None) -> int:
    return load().jm_noalloc_poll_error(_stream(stream))


def jm_noalloc_selftest_timeout(stream=None, check: bool = True) -> int:
    st = load().jm_noalloc_selftest_timeout(_stream(stream))
    if check:
        _check(st)
    return st


def jm_last_error() -> str:
    return load().jm_last_error().decode()


def jm_last_launch_count() -> int:
    return load().jm_last_launch_count()


def jm_last_kernel_name(index: int) -> str:
    return load().jm_last_kernel_name(index).decode()


_event_arr = None


def jm_set_kernel_events(handles) -> None:
    """Set (a sequence of raw cudaEvent_t handles) or clear (None) the per-kernel
    timing events."""
    global _event_arr
    if not handles:
        _event_arr = None
        _check(load().jm_set_kernel_events(None, 0))
        return
    _event_arr = (ctypes.c_void_p * len(handles))(*handles)
    _check(load().jm_set_kernel_events(_event_arr, len(handles)))

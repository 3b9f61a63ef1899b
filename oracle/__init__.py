"""fp64 CPU oracle of the Jamba Mamba-1 mixer core (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
cpu_baseline / reference legs of ``bench.py`` may use it; the product path
(``mamba_selective_scan_jamba_b200``) never imports it.  It shares no code
with the CUDA path.  The arithmetic lives in ``jmix_oracle.cpp``; this module
converts stored inputs (bf16 bit patterns or float32) exactly to float64 and
marshals arguments.

Pins (tests/test_oracle_pins.py) tie every function here to something other
than itself: closed forms of the scan, the brute-force "hidden attention"
matrix form, the split-and-carry invariant, step == forward, permutation and
batch independence, the conv impulse response, RMSNorm and softplus
identities, and the dt branch (RMSNorm scale invariance through the whole
mixer, dt_norm_w scaling equal to dtproj_w scaling, a one-hot dtproj_w that
turns dt_proj into a selection); tests/test_oracle_planted.py plants four
mistakes in a copy of the dt branch and checks that a pin fails for each.
What no pin can reach is agreement with trained Jamba checkpoints (the pages
print no weights or worked numbers), so the conv tap order stays a reading.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "jmix_oracle.cpp")
LIB = os.path.join(_HERE, "_build", "libjmix_oracle.so")

_P = ctypes.POINTER(ctypes.c_double)


class OrcDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("d_inner", ctypes.c_int64), ("d_state", ctypes.c_int64),
                ("d_conv", ctypes.c_int64), ("dt_rank", ctypes.c_int64),
                ("eps", ctypes.c_double), ("mirror_bf16", ctypes.c_int32),
                ("threads", ctypes.c_int32), ("zoh", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


def build(force: bool = False) -> str:
    """Compile the oracle with the host C++ compiler (IEEE double, no contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        os.makedirs(os.path.dirname(LIB), exist_ok=True)
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-O3", "-std=c++17", "-shared", "-fPIC", "-pthread",
                               "-ffp-contract=off", "-fno-fast-math", SRC, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


_lib = None


def load_library(path: str):
    """A ctypes handle on an oracle library built from this source (or, in the
    planted-mistake tests, from a mutated copy of it)."""
    lib = ctypes.CDLL(path)
    lib.orc_round_bf16.restype = ctypes.c_double
    lib.orc_round_bf16.argtypes = [ctypes.c_double]
    lib.orc_round_fp16.restype = ctypes.c_double
    lib.orc_round_fp16.argtypes = [ctypes.c_double]
    lib.orc_softplus1.restype = ctypes.c_double
    lib.orc_softplus1.argtypes = [ctypes.c_double]
    return lib


def _L():
    global _lib
    if _lib is None:
        build()
        _lib = load_library(LIB)
    return _lib


def _f64(a) -> np.ndarray:
    """Exact float64 copy of a stored tensor (uint16 = bf16 bit patterns)."""
    if a is None:
        return None
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = (a.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(_P)


def dims(batch, seqlen, d_inner, dt_rank, d_state=16, d_conv=4, eps=1e-6, mirror=False,
         threads=0, zoh=False) -> OrcDims:
    """zoh: discretise B by zero-order hold, (exp(delta A) - 1) / A * B, instead of delta B."""
    return OrcDims(batch, seqlen, d_inner, d_state, d_conv, dt_rank, eps, int(mirror), threads,
                   int(zoh), 0)


def dims_of(w, mirror=False, threads=0, batch=None, seqlen=None, zoh=None) -> OrcDims:
    """Oracle dims from a synth.Workload-like object (zoh defaults to the workload's)."""
    return dims(w.batch if batch is None else batch, w.seqlen if seqlen is None else seqlen,
                w.d_inner, w.dt_rank, w.d_state, w.d_conv, w.eps, mirror, threads,
                getattr(w, "zoh", False) if zoh is None else zoh)


_WNAMES = ("conv_w", "conv_b", "xproj_w", "dt_norm_w", "b_norm_w", "c_norm_w", "dtproj_w",
           "dt_bias", "A_log", "D")


def round_bf16(v: float) -> float:
    return _L().orc_round_bf16(float(v))


def round_fp16(v: float) -> float:
    return _L().orc_round_fp16(float(v))


def softplus1(v: float) -> float:
    return _L().orc_softplus1(float(v))


def conv(x, w, b, hist=None) -> np.ndarray:
    """Pre-activation causal conv of one sequence: x [L,d], w [d,K], b [d], hist [d,K-1]."""
    x, w, b, hist = _f64(x), _f64(w), _f64(b), _f64(hist)
    L, d = x.shape
    out = np.empty((L, d))
    _L().orc_conv(ctypes.c_int64(L), ctypes.c_int64(d), ctypes.c_int64(w.shape[1]), _p(x), _p(w),
                  _p(b), _p(hist), _p(out))
    return out


def silu(v) -> np.ndarray:
    v = _f64(v)
    out = np.empty_like(v)
    _L().orc_silu(ctypes.c_int64(v.size), _p(v), _p(out))
    return out


def softplus(v) -> np.ndarray:
    v = _f64(v)
    out = np.empty_like(v)
    _L().orc_softplus(ctypes.c_int64(v.size), _p(v), _p(out))
    return out


def rmsnorm(v, w, eps) -> np.ndarray:
    """RMSNorm over the last axis."""
    v, w = _f64(v), _f64(w)
    width = v.shape[-1]
    rows = v.size // width
    out = np.empty_like(v)
    _L().orc_rmsnorm(ctypes.c_int64(rows), ctypes.c_int64(width), ctypes.c_int64(width), _p(v),
                     _p(w), ctypes.c_double(eps), _p(out))
    return out


def scan(delta, A, Bm, Cm, u, D, h0=None, zoh=False):
    """Selective scan of one sequence.  delta, u [L,d]; A [d,N] (negative reals);
    Bm, Cm [L,N]; D [d]; h0 [d,N].  Returns (y_s [L,d], h_T [d,N]).  zoh: B
    discretised by zero-order hold instead of delta B."""
    delta, A, Bm, Cm, u, D, h0 = map(_f64, (delta, A, Bm, Cm, u, D, h0))
    L, d = delta.shape
    N = A.shape[1]
    y = np.empty((L, d))
    hT = np.empty((d, N))
    _L().orc_scan(ctypes.c_int64(L), ctypes.c_int64(d), ctypes.c_int64(N), _p(delta), _p(A),
                  _p(Bm), _p(Cm), _p(u), _p(D), _p(h0), _p(y), _p(hT), ctypes.c_int32(int(zoh)))
    return y, hT


def scan_bwd(delta, A_log, Bm, Cm, u, D, h0, gy):
    """Backward of the scan core of one sequence (Euler B), fp64.  delta, u, gy
    [L,d]; A_log [d,N]; Bm, Cm [L,N]; D [d]; h0 [d,N] or None.  Returns a dict of
    gradients: delta, u [L,d]; B, C [L,N]; A_log [d,N] (through A = -exp(A_log));
    D [d]; h0 [d,N]."""
    delta, A_log, Bm, Cm, u, D, h0, gy = map(_f64, (delta, A_log, Bm, Cm, u, D, h0, gy))
    L, d = delta.shape
    N = A_log.shape[1]
    A = -np.exp(A_log)
    out = {k: np.zeros(s) for k, s in (("delta", (L, d)), ("u", (L, d)), ("B", (L, N)),
                                        ("C", (L, N)), ("A", (d, N)), ("D", (d,)),
                                        ("h0", (d, N)))}
    _L().orc_scan_bwd(ctypes.c_int64(L), ctypes.c_int64(d), ctypes.c_int64(N), _p(delta), _p(A),
                      _p(Bm), _p(Cm), _p(u), _p(D), _p(h0), _p(gy), _p(out["delta"]),
                      _p(out["u"]), _p(out["B"]), _p(out["C"]), _p(out["A"]), _p(out["D"]),
                      _p(out["h0"]))
    out["A_log"] = out.pop("A") * A          # dA/dA_log = A
    return out


def mixer_fwd(m: OrcDims, x, z, weights: Dict[str, np.ndarray], init_conv_state=None,
              init_ssm_state=None, channels: Optional[Sequence[int]] = None):
    """Mixer forward.  Returns (y [B,L,d or nch], final_state [B,d or nch,N],
    final_conv [B,d or nch,K-1]) in float64.  With ``channels``, the front end
    still runs over every channel but only the chosen channels are scanned, and
    x is read in its stored form (no float64 copy of a full-size x)."""
    B, L, d, N, K = m.batch, m.seqlen, m.d_inner, m.d_state, m.d_conv
    assert x.shape == (B, L, d) and z.shape == (B, L, d)
    W = [_f64(weights[k]) for k in _WNAMES]
    ic, iss = _f64(init_conv_state), _f64(init_ssm_state)
    if channels is None:
        x, z = _f64(x), _f64(z)
        y = np.empty((B, L, d))
        fs = np.empty((B, d, N))
        fc = np.empty((B, d, K - 1))
        _L().orc_mixer_fwd(ctypes.byref(m), _p(x), _p(z), *[_p(a) for a in W], _p(ic), _p(iss),
                           _p(y), _p(fs), _p(fc))
        return y, fs, fc
    ch = np.ascontiguousarray(channels, dtype=np.int64)
    nch = ch.size
    xs = np.ascontiguousarray(x)
    xkind = {np.dtype(np.uint16): 1, np.dtype(np.float32): 2}.get(xs.dtype, 0)
    if xkind == 0:
        xs = np.ascontiguousarray(xs, dtype=np.float64)
    zsel = _f64(np.asarray(z)[:, :, ch])
    y = np.empty((B, L, nch))
    fs = np.empty((B, nch, N))
    fc = np.empty((B, nch, K - 1))
    _L().orc_mixer_fwd_channels(ctypes.byref(m), xs.ctypes.data_as(ctypes.c_void_p),
                                ctypes.c_int32(xkind), _p(zsel), *[_p(a) for a in W], _p(ic),
                                _p(iss), ctypes.c_int64(nch),
                                ch.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), _p(y), _p(fs),
                                _p(fc))
    return y, fs, fc


def _round_bf16_via_f32(a: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (nearest even) -> bf16 (nearest even), as a float32-accumulating
    GEMM that stores bf16 rounds its outputs (finite values)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def layer_fwd(m: OrcDims, hidden, in_proj_w, out_proj_w, weights: Dict[str, np.ndarray],
              init_conv_state=None, init_ssm_state=None, round_xz_bf16: bool = False):
    """The full Mamba layer around the mixer core (TransformerLens "Jamba" adapter
    page, "Architecture overview": in_proj / conv1d / x_proj / dt_proj / out_proj):
    [x | z] = hidden . in_proj_w^T, the mixer core, out = y . out_proj_w^T.  fp64
    matrix products.  round_xz_bf16 rounds x and z to bf16 (nearest even) before the
    mixer, as a bf16 layer stores them.  Returns (out [B,L,d_model], final_state)."""
    h = _f64(hidden)
    wi, wo = _f64(in_proj_w), _f64(out_proj_w)
    d = m.d_inner
    xz = h @ wi.T
    x, z = np.ascontiguousarray(xz[..., :d]), np.ascontiguousarray(xz[..., d:])
    if round_xz_bf16:
        x, z = _round_bf16_via_f32(x), _round_bf16_via_f32(z)
    y, fs, _ = mixer_fwd(m, x, z, weights, init_conv_state, init_ssm_state)
    return y @ wo.T, fs


def mixer_step(m: OrcDims, x_t, z_t, conv_state, ssm_state, weights: Dict[str, np.ndarray]):
    """One decode step for every sequence.  Returns (y_t [B,d], conv_state', ssm_state')
    in float64; the inputs are not modified."""
    B, d, N, K = m.batch, m.d_inner, m.d_state, m.d_conv
    W = [_f64(weights[k]) for k in _WNAMES]
    x_t, z_t = _f64(x_t), _f64(z_t)
    cs = _f64(conv_state).copy()
    ss = _f64(ssm_state).copy()
    y = np.empty((B, d))
    _L().orc_mixer_step(ctypes.byref(m), _p(x_t), _p(z_t), _p(cs), _p(ss), *[_p(a) for a in W],
                        _p(y))
    return y, cs, ss

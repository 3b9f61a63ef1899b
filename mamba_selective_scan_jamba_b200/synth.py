"""Seeded synthetic inputs for the Jamba Mamba-1 mixer core.

This module is the single source of inputs for both the CUDA path and the
fp64 oracle.  It holds none of the mixer's arithmetic: only a counter-based
random generator, the bf16 storage encoding, and the workload recipes (shapes
and value distributions) of the five Jamba-shaped workloads.

Generator
---------
SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014): the i-th draw of a stream with seed ``s`` is
``mix(s + (i + 1) * 0x9E3779B97F4A7C15)``.  A uniform double in [0, 1) keeps the
top 53 bits.  Normals use the Box-Muller transform on the pair of uniforms
(2k, 2k+1).  Every tensor has its own stream, seeded with
``mix(workload_seed XOR (tensor_id << 32))``.  The bulk generator is C
(``csrc/synth_gen.c``, threaded over index ranges); ``np_uniform`` /
``np_normal`` restate it in numpy so tests can cross-check it.

Value recipe (Jamba v0.1 mixer: d_inner 8192, d_state 16, d_conv 4,
dt_rank ceil(4096/16) = 256, as listed on the llm-architectures-explained
"Jamba v0.1" page, "Every architecture field" table):

* x, z ~ N(0, 1); conv_w ~ U(-1/2, 1/2); conv_b = 0
* xproj_w ~ N(0, 1/d_inner); dtproj_w ~ N(0, 1/dt_rank)  (second argument = variance)
* dt log-uniform in [1e-3, 1e-1] ([1e-4, 1e-1] for the 256K workload),
  dt_bias = log(expm1(dt)) so that softplus(dt_bias) = dt
* A_log[c, n] = log(n + 1) (the initialisation of the aifetchly guide's toy
  SSM, "Hands-On Implementation"); D = 1; RMSNorm weights 1; eps 1e-6
* decode: conv_state ~ N(0, 1), ssm_state ~ N(0, 0.1), a fresh (x_t, z_t) per step

``extra=True`` replaces the degenerate constants (conv_b = 0, norm weights 1,
D = 1, structured A_log, zero initial states) with random values so that
parity tests see every term.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, replace
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SYNTH_LIB = os.path.join(_HERE, "_build", "libjmix_synth.so")

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

# tensor ids used to derive per-tensor streams
TID = dict(x=1, z=2, conv_w=3, conv_b=4, xproj_w=5, dtproj_w=6, dt=7,
           dt_norm_w=8, b_norm_w=9, c_norm_w=10, D=11, A_log=12,
           init_conv_state=13, init_ssm_state=14, conv_state=15, ssm_state=16)
TID_LAYER = dict(hidden=20, in_proj_w=21, out_proj_w=22)  # the full layer's extra tensors
TID_XT = 1000   # + step index
TID_ZT = 2000   # + step index

_OUT = {"f64": 0, "f32": 1, "bf16": 2}
_lib = None


def _clib():
    global _lib
    if _lib is None:
        if not os.path.exists(SYNTH_LIB):
            from . import build as _b
            _b.build_synth()
        lib = ctypes.CDLL(SYNTH_LIB)
        for fn in (lib.jms_uniform, lib.jms_normal):
            fn.restype = None
            fn.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                           ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
        _lib = lib
    return _lib


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def mix64(v: int) -> int:
    """SplitMix64 finaliser of one 64-bit integer (used to derive stream seeds)."""
    with np.errstate(over="ignore"):
        return int(_mix(np.array([v & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0])


def stream_seed(workload_seed: int, tensor_id: int) -> int:
    return mix64((workload_seed ^ (tensor_id << 32)) & 0xFFFFFFFFFFFFFFFF)


def _gen(kind: str, seed: int, n: int, start: int, scale: float, shift: float, out: str):
    dt = {"f64": np.float64, "f32": np.float32, "bf16": np.uint16}[out]
    arr = np.empty(n, dtype=dt)
    if n:
        fn = _clib().jms_uniform if kind == "u" else _clib().jms_normal
        fn(seed & 0xFFFFFFFFFFFFFFFF, start, n, scale, shift, _OUT[out],
           arr.ctypes.data_as(ctypes.c_void_p), 0)
    return arr


def uniform(seed: int, n: int, start: int = 0, scale: float = 1.0, shift: float = 0.0,
            out: str = "f64") -> np.ndarray:
    """scale * U[start .. start+n) + shift, U uniform in [0, 1)."""
    return _gen("u", seed, n, start, scale, shift, out)


def normal(seed: int, n: int, std: float = 1.0, start: int = 0, out: str = "f64") -> np.ndarray:
    """std * Normal[start .. start+n)."""
    return _gen("n", seed, n, start, std, 0.0, out)


def np_uniform(seed: int, n: int, start: int = 0) -> np.ndarray:
    """numpy restatement of ``uniform`` (cross-check of the C generator)."""
    out = np.empty(n, dtype=np.float64)
    s = np.uint64(seed & 0xFFFFFFFFFFFFFFFF)
    with np.errstate(over="ignore"):
        for a in range(0, n, _CHUNK):
            b = min(n, a + _CHUNK)
            idx = np.arange(start + a + 1, start + b + 1, dtype=np.uint64)
            z = _mix(s + idx * _GAMMA)
            out[a:b] = (z >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    return out


def np_normal(seed: int, n: int, std: float = 1.0) -> np.ndarray:
    """numpy restatement of ``normal`` from draw 0 (cross-check of the C generator)."""
    npairs = (n + 1) // 2
    u = np_uniform(seed, 2 * npairs)
    r = np.sqrt(-2.0 * np.log1p(-u[0::2]))
    th = (2.0 * math.pi) * u[1::2]
    blk = np.empty(2 * npairs, dtype=np.float64)
    blk[0::2] = r * np.cos(th)
    blk[1::2] = r * np.sin(th)
    return blk[:n] * std


# ---------------------------------------------------------------- bf16 storage
def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); uint16 bit patterns."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def storage_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 view of a stored tensor (bf16 bit patterns or float32)."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


# -------------------------------------------------------------- workload recipes
@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    d_inner: int
    dt_rank: int
    io: str                      # "f32" or "bf16"
    seed: int
    d_state: int = 16
    d_conv: int = 4
    eps: float = 1e-6
    dt_min: float = 1e-3
    dt_max: float = 1e-1
    zoh: bool = False            # B discretised by zero-order hold (else delta B)
    steps: int = 0               # decode workloads: number of consecutive steps
    extra: bool = False          # random conv_b / norm weights / D / A_log / initial states

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    @property
    def proj(self) -> int:
        return self.dt_rank + 2 * self.d_state

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload("tiny_fp32", 1, 64, 128, 8, "f32", seed=1),
    "jamba_b1_l4096": Workload("jamba_b1_l4096", 1, 4096, 8192, 256, "bf16", seed=2),
    "jamba_b8_l4096": Workload("jamba_b8_l4096", 8, 4096, 8192, 256, "bf16", seed=3),
    "jamba_b1_l262144": Workload("jamba_b1_l262144", 1, 262144, 8192, 256, "bf16", seed=4,
                                 dt_min=1e-4),
    "jamba_decode_b256": Workload("jamba_decode_b256", 256, 1, 8192, 256, "bf16", seed=5,
                                  steps=64),
}


def _io(w: Workload) -> str:
    return "bf16" if w.io == "bf16" else "f32"


def _const(v: float, shape, io: str) -> np.ndarray:
    a = np.full(shape, v, dtype=np.float32)
    return f32_to_bf16_bits(a) if io == "bf16" else a


def make_weights(w: Workload) -> Dict[str, np.ndarray]:
    """Per-layer parameters.  Matrices, conv and norm weights use the I/O dtype;
    dt_bias, A_log and D are float32."""
    d, R, N, K, P = w.d_inner, w.dt_rank, w.d_state, w.d_conv, w.proj
    io = _io(w)
    s = lambda name: stream_seed(w.seed, TID[name])
    out: Dict[str, np.ndarray] = {}
    out["conv_w"] = uniform(s("conv_w"), d * K, shift=-0.5, out=io).reshape(d, K)
    out["conv_b"] = (uniform(s("conv_b"), d, shift=-0.5, out=io) if w.extra
                     else _const(0.0, (d,), io))
    out["xproj_w"] = normal(s("xproj_w"), P * d, 1.0 / math.sqrt(d), out=io).reshape(P, d)
    out["dtproj_w"] = normal(s("dtproj_w"), d * R, 1.0 / math.sqrt(R), out=io).reshape(d, R)
    if w.extra:
        out["dt_norm_w"] = uniform(s("dt_norm_w"), R, shift=0.5, out=io)
        out["b_norm_w"] = uniform(s("b_norm_w"), N, shift=0.5, out=io)
        out["c_norm_w"] = uniform(s("c_norm_w"), N, shift=0.5, out=io)
    else:
        out["dt_norm_w"] = _const(1.0, (R,), io)
        out["b_norm_w"] = _const(1.0, (N,), io)
        out["c_norm_w"] = _const(1.0, (N,), io)
    lo, hi = math.log(w.dt_min), math.log(w.dt_max)
    dt = np.exp(uniform(s("dt"), d, scale=hi - lo, shift=lo))
    out["dt_bias"] = np.log(np.expm1(dt)).astype(np.float32)
    if w.extra:
        # A_n = -exp(A_log) spread log-uniformly over [1/4, 16): no structure across n
        out["A_log"] = uniform(s("A_log"), d * N, scale=math.log(64.0), shift=math.log(0.25),
                               out="f32").reshape(d, N)
        out["D"] = normal(s("D"), d, out="f32")
    else:
        out["A_log"] = np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)),
                               (d, 1)).astype(np.float32)
        out["D"] = np.ones(d, dtype=np.float32)
    return out


def make_activations(w: Workload, batch_lo: int = 0, batch_hi: Optional[int] = None
                     ) -> Dict[str, np.ndarray]:
    """x, z [b, L, d] for sequences batch_lo..batch_hi-1 (a sequence's values do not
    depend on the slice), plus the initial states when ``w.extra``."""
    hi = w.batch if batch_hi is None else batch_hi
    nb = hi - batch_lo
    d, L, N, K = w.d_inner, w.seqlen, w.d_state, w.d_conv
    io = _io(w)
    per = L * d
    out: Dict[str, np.ndarray] = {}
    for name in ("x", "z"):
        out[name] = normal(stream_seed(w.seed, TID[name]), nb * per, start=batch_lo * per,
                           out=io).reshape(nb, L, d)
    if w.extra:
        out["init_conv_state"] = normal(stream_seed(w.seed, TID["init_conv_state"]),
                                        nb * d * (K - 1), start=batch_lo * d * (K - 1),
                                        out=io).reshape(nb, d, K - 1)
        out["init_ssm_state"] = normal(stream_seed(w.seed, TID["init_ssm_state"]), nb * d * N,
                                       math.sqrt(0.1), start=batch_lo * d * N,
                                       out="f32").reshape(nb, d, N)
    return out


def make_layer(w: Workload, d_model: int) -> Dict[str, np.ndarray]:
    """The full Mamba layer's extra tensors around the mixer core: hidden [B, L,
    d_model] ~ N(0, 1); in_proj_w [2 d_inner, d_model] ~ N(0, 1/d_model) (rows
    0..d_inner-1 give x, the rest z); out_proj_w [d_model, d_inner] ~ N(0, 1/d_inner).
    I/O dtype."""
    d, io = w.d_inner, _io(w)
    s = lambda name: stream_seed(w.seed, TID_LAYER[name])
    return {"hidden": normal(s("hidden"), w.batch * w.seqlen * d_model, out=io)
                      .reshape(w.batch, w.seqlen, d_model),
            "in_proj_w": normal(s("in_proj_w"), 2 * d * d_model, 1.0 / math.sqrt(d_model),
                                out=io).reshape(2 * d, d_model),
            "out_proj_w": normal(s("out_proj_w"), d_model * d, 1.0 / math.sqrt(d),
                                 out=io).reshape(d_model, d)}


def make_decode_state(w: Workload) -> Dict[str, np.ndarray]:
    """Cached states for the decode workload: conv_state [B, d, d_conv-1] (I/O dtype,
    oldest tap first), ssm_state [B, d, N] float32."""
    B, d, N, K = w.batch, w.d_inner, w.d_state, w.d_conv
    return {"conv_state": normal(stream_seed(w.seed, TID["conv_state"]), B * d * (K - 1),
                                 out=_io(w)).reshape(B, d, K - 1),
            "ssm_state": normal(stream_seed(w.seed, TID["ssm_state"]), B * d * N,
                                math.sqrt(0.1), out="f32").reshape(B, d, N)}


def make_decode_token(w: Workload, step: int) -> Dict[str, np.ndarray]:
    """Fresh (x_t, z_t) [B, d] for one decode step."""
    B, d = w.batch, w.d_inner
    return {"x_t": normal(stream_seed(w.seed, TID_XT + step), B * d, out=_io(w)).reshape(B, d),
            "z_t": normal(stream_seed(w.seed, TID_ZT + step), B * d, out=_io(w)).reshape(B, d)}

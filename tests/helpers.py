"""Shared helpers of the parity tests: run the CUDA path through the C ABI and
compare with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

import oracle
from mamba_selective_scan_jamba_b200 import synth

# Gates (the mixer's stated tolerances):
#   float32 io: |y - y_ref| <= 1e-4 max(1, |y_ref|), states the same, exact oracle
#   bf16 io:    |y - y_ref| <= 2e-2 max(1, |y_ref|) against the exact oracle;
#               final SSM state <= 1e-4 max(1, |ref|) against the mirror-rounded oracle
TOL = {"f32": dict(y=1e-4, state=1e-4), "bf16": dict(y=2e-2, state=1e-4, y_mirror=1e-2)}


def f64(a: np.ndarray) -> np.ndarray:
    return synth.storage_to_f64(a)


def max_scaled_err(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.size == 0:
        return 0.0
    assert np.isfinite(got).all(), "non-finite output"
    return float((np.abs(got - ref) / np.maximum(1.0, np.abs(ref))).max())


def gpu_fwd(w: synth.Workload, W: Dict[str, np.ndarray], A: Dict[str, np.ndarray],
            use_init: bool = True, want_conv: bool = True, stream=None):
    """Run jm_mixer_fwd on cuda:0; returns host (y, final_state, final_conv) in stored dtypes."""
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    dev = "cuda"
    Wd = devio.weights_to_device(W, dev)
    x = devio.to_device(A["x"], dev)
    z = devio.to_device(A["z"], dev)
    y = torch.empty_like(x)
    fs = torch.empty((w.batch, w.d_inner, w.d_state), dtype=torch.float32, device=dev)
    ic = devio.to_device(A["init_conv_state"], dev) if use_init and "init_conv_state" in A else None
    iss = devio.to_device(A["init_ssm_state"], dev) if use_init and "init_ssm_state" in A else None
    fc = (torch.empty((w.batch, w.d_inner, w.d_conv - 1), dtype=x.dtype, device=dev)
          if want_conv else None)
    d = devio.dims_of(w)
    nbytes = jmix.jm_mixer_fwd_workspace_size(d)
    ws = devio.workspace(nbytes, dev)
    jmix.jm_mixer_fwd(d, x, z, Wd, y, fs, ws, nbytes, ic, iss, fc, stream=stream)
    assert jmix.jm_poll_error(ws) == jmix.JM_OK, jmix.jm_last_error()
    torch.cuda.synchronize()
    return devio.to_host(y), devio.to_host(fs), (devio.to_host(fc) if fc is not None else None)


def check_fwd(w: synth.Workload, channels: Optional[Sequence[int]] = None, use_init=True,
              threads: int = 0):
    """GPU forward vs oracle on one workload; returns the measured errors."""
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    y, fs, fc = gpu_fwd(w, W, A, use_init)
    ic = A.get("init_conv_state") if use_init else None
    iss = A.get("init_ssm_state") if use_init else None
    tol = TOL[w.io]
    errs = {}
    if w.io == "f32":
        yr, fsr, fcr = oracle.mixer_fwd(oracle.dims_of(w, threads=threads), A["x"], A["z"], W,
                                        ic, iss, channels=channels)
        sel = slice(None) if channels is None else list(channels)
        errs["y"] = max_scaled_err(y[:, :, sel], yr)
        errs["state"] = max_scaled_err(fs[:, sel], fsr)
        assert errs["y"] <= tol["y"], errs
        assert errs["state"] <= tol["state"], errs
    else:
        yr, _, fcr = oracle.mixer_fwd(oracle.dims_of(w, threads=threads), A["x"], A["z"], W, ic,
                                      iss, channels=channels)
        ym, fsm, _ = oracle.mixer_fwd(oracle.dims_of(w, mirror=True, threads=threads), A["x"],
                                      A["z"], W, ic, iss, channels=channels)
        sel = slice(None) if channels is None else list(channels)
        yg = f64(y)[:, :, sel]
        errs["y"] = max_scaled_err(yg, yr)
        errs["y_mirror"] = max_scaled_err(yg, ym)
        errs["state"] = max_scaled_err(fs[:, sel], fsm)
        assert errs["y"] <= tol["y"], errs
        assert errs["y_mirror"] <= tol["y_mirror"], errs
        assert errs["state"] <= tol["state"], errs
    sel = slice(None) if channels is None else list(channels)
    np.testing.assert_array_equal(f64(fc)[:, sel], fcr)   # conv state: exact copy of inputs
    return errs

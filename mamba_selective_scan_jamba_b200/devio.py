"""Device-memory plumbing for callers of libjmix: torch allocates, libjmix computes.

Stored tensors use numpy uint16 for bf16 bit patterns and float32 otherwise;
on the device they become torch.bfloat16 / torch.float32 tensors with the same
bytes.  Nothing here computes any part of the mixer.
"""
from __future__ import annotations

from typing import Dict, Mapping

import numpy as np
import torch

from . import jmix


def to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def to_host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_pinned(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).pin_memory().view(torch.bfloat16)
    else:
        t = torch.from_numpy(a).pin_memory()
    return t


def io_dtype(io: str) -> torch.dtype:
    return torch.bfloat16 if io == "bf16" else torch.float32


def weights_to_device(W: Mapping[str, np.ndarray], device="cuda") -> Dict[str, torch.Tensor]:
    return {k: to_device(W[k], device) for k in jmix.WEIGHT_NAMES}


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device buffer of at least nbytes."""
    t = torch.empty(max(int(nbytes), 256) + 256, dtype=torch.uint8, device=device)
    off = (-t.data_ptr()) % 256
    return t[off:off + max(int(nbytes), 256)]


def dims_of(w, batch=None, seqlen=None) -> jmix.jm_dims:
    """jm_dims for a synth.Workload."""
    return jmix.dims(w.batch if batch is None else batch, w.seqlen if seqlen is None else seqlen,
                     w.d_inner, w.dt_rank, jmix.JM_BF16 if w.io == "bf16" else jmix.JM_F32,
                     w.eps, w.d_state, w.d_conv, getattr(w, "zoh", False))

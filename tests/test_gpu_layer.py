"""jm_layer_fwd: in_proj -> mixer core -> out_proj on cuda:0, against the fp64
layer oracle (matrix products in fp64 around the mixer oracle).  The cases
cover the tcgen05 GEMM's edges: ragged row tiles, one partial row tile, and
enough tiles that every persistent CTA runs many, alternating its two TMEM
accumulators and wrapping its stage ring.

Gates: out within 2e-2 max(1, |ref|) of the exact oracle (as y); the final
SSM state within 2e-3 max(1, |ref|) of the mirror oracle fed with x, z rounded
to bf16.  The looser state gate is derived: x and z come from a float32-
accumulating GEMM, so a few of their bf16 roundings fall on the other side of
the oracle's (one bf16 ulp, 2^-8 relative, of one x value moves a state by at
most about 2^-8 of one token's delta*B*u share); the mixer's own 1e-4 state gate
applies to the mixer tests.
"""
import numpy as np
import pytest

import oracle
from mamba_selective_scan_jamba_b200 import synth
from tests.helpers import f64, max_scaled_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,L,d,R,d_model", [
    (2, 130, 512, 32, 256),       # ragged row tiles; in_proj N = 1024, out_proj N = 256
    (1, 64, 8192, 256, 4096),     # Jamba's d_model / d_inner, a single partial row tile
    (2, 4096, 4096, 128, 2048),   # many tiles per CTA: 2048 in_proj and 512 out_proj tiles
])
def test_layer_matches_oracle(B, L, d, R, d_model):
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    w = synth.Workload("layer", B, L, d, R, "bf16", seed=23, extra=(d != 8192))
    W = synth.make_weights(w)
    LW = synth.make_layer(w, d_model)
    A = synth.make_activations(w)
    ic, iss = A.get("init_conv_state"), A.get("init_ssm_state")
    Wd = devio.weights_to_device(W)
    hid = devio.to_device(LW["hidden"])
    out = torch.empty_like(hid)
    fs = torch.empty((B, d, 16), dtype=torch.float32, device="cuda")
    dm = devio.dims_of(w)
    n = jmix.jm_layer_fwd_workspace_size(dm, d_model)
    ws = devio.workspace(n)
    jmix.jm_layer_fwd(dm, d_model, hid, devio.to_device(LW["in_proj_w"]), Wd,
                      devio.to_device(LW["out_proj_w"]), out, fs, ws, n,
                      None if ic is None else devio.to_device(ic),
                      None if iss is None else devio.to_device(iss))
    assert jmix.jm_poll_error(ws) == jmix.JM_OK, jmix.jm_last_error()
    torch.cuda.synchronize()
    ref, _ = oracle.layer_fwd(oracle.dims_of(w), LW["hidden"], LW["in_proj_w"],
                              LW["out_proj_w"], W, ic, iss)
    _, fsm = oracle.layer_fwd(oracle.dims_of(w, mirror=True), LW["hidden"], LW["in_proj_w"],
                              LW["out_proj_w"], W, ic, iss, round_xz_bf16=True)
    assert max_scaled_err(f64(devio.to_host(out)), ref) <= 2e-2
    assert max_scaled_err(devio.to_host(fs), fsm) <= 2e-3

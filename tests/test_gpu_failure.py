"""Failure detection and unwritten-read checks on cuda:0, with no fault.

* A bounded device-side wait that nothing satisfies gives up, records its site,
  and the host reads JM_ERR_TIMEOUT; the context then runs a forward normally.
* Every call writes each workspace byte it reads: a workspace filled with NaN
  bit patterns gives the same bits as a zero-filled one (forward, packed
  batch, decode step).
"""
import numpy as np
import pytest

from mamba_selective_scan_jamba_b200 import synth
from tests.helpers import check_fwd

pytestmark = pytest.mark.gpu


def test_timeout_is_reported_and_the_context_survives():
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    ws = devio.workspace(256)
    jmix.jm_selftest_timeout(ws, 256)
    assert jmix.jm_poll_error(ws) == jmix.JM_ERR_TIMEOUT
    assert "site 99" in jmix.jm_last_error()
    torch.cuda.synchronize()
    check_fwd(synth.Workload("after_timeout", 2, 70, 256, 32, "bf16", seed=4, extra=True))


def _fill(ws, byte):
    ws.fill_(byte)


@pytest.mark.parametrize("mode", ["fwd", "varlen", "step"])
def test_nan_poisoned_workspace_gives_the_same_bits(mode):
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    w = synth.Workload("poison", 3, 300 if mode != "step" else 1, 384, 64, "bf16", seed=6,
                       extra=True)
    W = devio.weights_to_device(synth.make_weights(w))
    A = synth.make_activations(w)
    x, z = devio.to_device(A["x"]), devio.to_device(A["z"])
    ic, iss = devio.to_device(A["init_conv_state"]), devio.to_device(A["init_ssm_state"])
    outs = []
    for byte in (0x00, 0xFF):          # 0xFFFF... is a NaN in every float format here
        y = torch.empty_like(x)
        fs = torch.empty((w.batch, w.d_inner, 16), dtype=torch.float32, device="cuda")
        fc = torch.empty_like(ic)
        if mode == "fwd":
            d = devio.dims_of(w)
            n = jmix.jm_mixer_fwd_workspace_size(d)
            ws = devio.workspace(n)
            _fill(ws, byte)
            jmix.jm_mixer_fwd(d, x, z, W, y, fs, ws, n, ic, iss, fc)
        elif mode == "varlen":
            d = jmix.dims(w.batch, w.batch * w.seqlen, w.d_inner, w.dt_rank)
            n = jmix.jm_mixer_fwd_varlen_workspace_size(d)
            ws = devio.workspace(n)
            _fill(ws, byte)
            cu = torch.tensor([0, 300, 600, 900], dtype=torch.int32, device="cuda")
            jmix.jm_mixer_fwd_varlen(d, cu, x.view(-1, w.d_inner), z.view(-1, w.d_inner), W,
                                     y.view(-1, w.d_inner), fs, ws, n, ic, iss, fc)
        else:
            d = devio.dims_of(w)
            n = jmix.jm_mixer_step_workspace_size(d)
            ws = devio.workspace(n)
            _fill(ws, byte)
            cs, ss = ic.clone(), iss.clone()
            jmix.jm_mixer_step(d, x.view(w.batch, w.d_inner), z.view(w.batch, w.d_inner), cs, ss,
                               W, y.view(w.batch, w.d_inner), ws, n)
            fs, fc = ss, cs
        assert jmix.jm_poll_error(ws) == jmix.JM_OK, jmix.jm_last_error()
        torch.cuda.synchronize()
        outs.append((devio.to_host(y), devio.to_host(fs), devio.to_host(fc)))
    for a, b in zip(outs[0], outs[1]):
        np.testing.assert_array_equal(a, b)

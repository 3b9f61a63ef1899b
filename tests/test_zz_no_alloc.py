"""jm_mixer_step_noalloc: the decode step for callers that cannot allocate
device memory (engines that give plug-ins no allocator).  Its scratch is a static device array inside libjmix; these tests
check it against jm_mixer_step with a caller workspace, on two steps in a row.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest

from mamba_selective_scan_jamba_b200 import build, jmix, synth
from tests.helpers import f64, max_scaled_err


def test_noalloc_rejects_steps_beyond_its_buffer():
    """Needs no GPU: the size check runs before any CUDA call."""
    build.build_libjmix()
    FAKE = 1 << 40
    W = {k: FAKE for k in jmix.WEIGHT_NAMES}
    d = jmix.dims(4096, 1, 8192, 256)          # ~270 MiB of scratch, far above 32 MiB
    st = jmix.jm_mixer_step_noalloc(d, FAKE, FAKE, FAKE, FAKE, W, FAKE + (1 << 36), stream=0,
                                    check=False)
    assert st == jmix.JM_ERR_UNSUPPORTED
    assert "static buffer" in jmix.jm_last_error()
    bad = jmix.dims(4, 1, 8192, 256, d_state=8)
    st = jmix.jm_mixer_step_noalloc(bad, FAKE, FAKE, FAKE, FAKE, W, FAKE + (1 << 36), stream=0,
                                    check=False)
    assert st == jmix.JM_ERR_UNSUPPORTED and "d_state" in jmix.jm_last_error()


@pytest.mark.gpu
@pytest.mark.parametrize("B,d,R,io", [(4, 1024, 64, "bf16"), (3, 256, 16, "f32"),
                                      (256, 8192, 256, "bf16")])
def test_noalloc_step_matches_workspace_step(B, d, R, io):
    import torch
    from mamba_selective_scan_jamba_b200 import devio
    w = synth.Workload("noalloc", B, 1, d, R, io, seed=31, extra=True, steps=2)
    W = synth.make_weights(w)
    S = synth.make_decode_state(w)
    Wd = devio.weights_to_device(W)
    cs_a, ss_a = devio.to_device(S["conv_state"]), devio.to_device(S["ssm_state"])
    cs_b, ss_b = cs_a.clone(), ss_a.clone()
    dm = devio.dims_of(w)
    n = jmix.jm_mixer_step_workspace_size(dm)
    ws = devio.workspace(n)
    for step in range(2):
        tok = synth.make_decode_token(w, step)
        xt, zt = devio.to_device(tok["x_t"]), devio.to_device(tok["z_t"])
        y_a, y_b = torch.empty_like(xt), torch.empty_like(xt)
        ws.fill_(0xFF)   # NaN in every float format: a read of stale scratch would show
        jmix.jm_mixer_step(dm, xt, zt, cs_a, ss_a, Wd, y_a, ws, n)
        jmix.jm_mixer_step_noalloc(dm, xt, zt, cs_b, ss_b, Wd, y_b)
        torch.cuda.synchronize()
        assert jmix.jm_noalloc_poll_error() == jmix.JM_OK, jmix.jm_last_error()
        # the same kernels with the same scratch layout: the same bits, within
        # any tolerance the parity tests use
        np.testing.assert_array_equal(devio.to_host(y_b), devio.to_host(y_a))
        np.testing.assert_array_equal(devio.to_host(ss_b), devio.to_host(ss_a))
        np.testing.assert_array_equal(devio.to_host(cs_b), devio.to_host(cs_a))
        assert max_scaled_err(f64(devio.to_host(y_b)), f64(devio.to_host(y_a))) == 0.0


@pytest.mark.gpu
def test_noalloc_poll_reports_a_wait_that_ran_out():
    """A bounded wait that runs out inside the static array's header is reported by
    jm_noalloc_poll_error (there is no caller workspace for jm_poll_error to read),
    and the next step clears it."""
    import torch
    from mamba_selective_scan_jamba_b200 import devio
    jmix.jm_noalloc_selftest_timeout()
    assert jmix.jm_noalloc_poll_error() == jmix.JM_ERR_TIMEOUT
    assert "site 99" in jmix.jm_last_error()
    w = synth.Workload("noalloc_after", 2, 1, 256, 16, "bf16", seed=33, extra=True, steps=1)
    W = synth.make_weights(w)
    S = synth.make_decode_state(w)
    tok = synth.make_decode_token(w, 0)
    Wd = devio.weights_to_device(W)
    cs, ss = devio.to_device(S["conv_state"]), devio.to_device(S["ssm_state"])
    xt, zt = devio.to_device(tok["x_t"]), devio.to_device(tok["z_t"])
    yt = torch.empty_like(xt)
    jmix.jm_mixer_step_noalloc(devio.dims_of(w), xt, zt, cs, ss, Wd, yt)
    assert jmix.jm_noalloc_poll_error() == jmix.JM_OK, jmix.jm_last_error()
    assert torch.isfinite(yt.float()).all()

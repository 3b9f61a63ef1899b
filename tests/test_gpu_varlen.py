"""jm_mixer_fwd_varlen: a packed batch of variable-length sequences (serving
prefill) on cuda:0, against the fp64 oracle run sequence by sequence.

Every sequence has its own seeded activations and initial states; the weights
are shared.  Lengths include 0 (an empty sequence: its final states are its
initial ones), 1, 2 and 3 (history only from the cached conv state) and
lengths that end mid-chunk, so sequence starts fall inside conv token groups
and scan chunks.
"""
import numpy as np
import pytest

import oracle
from mamba_selective_scan_jamba_b200 import synth
from tests.helpers import TOL, f64, max_scaled_err

pytestmark = pytest.mark.gpu


def _packed_inputs(base: synth.Workload, lengths):
    W = synth.make_weights(base)
    per = []
    for b, L in enumerate(lengths):
        wb = base.with_(batch=1, seqlen=max(L, 1), seed=base.seed * 1000 + b)
        A = synth.make_activations(wb)
        if L == 0:
            A = dict(A, x=A["x"][:, :0], z=A["z"][:, :0])
        per.append(A)
    x = np.concatenate([A["x"][0] for A in per], 0)
    z = np.concatenate([A["z"][0] for A in per], 0)
    ic = np.concatenate([A["init_conv_state"] for A in per], 0)
    iss = np.concatenate([A["init_ssm_state"] for A in per], 0)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return W, per, x, z, ic, iss, cu


def _run_varlen(base, lengths, x, z, W, ic, iss, cu):
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    B, T = len(lengths), x.shape[0]   # the token count comes from the data, not from cu
    d = jmix.dims(B, T, base.d_inner, base.dt_rank, jmix.JM_BF16, base.eps)
    Wd = devio.weights_to_device(W)
    xd, zd = devio.to_device(x), devio.to_device(z)
    y = torch.empty_like(xd)
    fs = torch.empty((B, base.d_inner, 16), dtype=torch.float32, device="cuda")
    fc = torch.empty((B, base.d_inner, 3), dtype=torch.bfloat16, device="cuda")
    n = jmix.jm_mixer_fwd_varlen_workspace_size(d)
    ws = devio.workspace(n)
    cud = torch.from_numpy(cu).cuda()
    jmix.jm_mixer_fwd_varlen(d, cud, xd, zd, Wd, y, fs, ws, n, devio.to_device(ic),
                             devio.to_device(iss), fc)
    status = jmix.jm_poll_error(ws)
    torch.cuda.synchronize()
    return status, devio.to_host(y), devio.to_host(fs), devio.to_host(fc)


@pytest.mark.parametrize("lengths,d,R", [
    ([1, 2, 3, 40, 300, 0, 1000, 77, 5], 256, 64),
    ([4096, 17, 2050], 1024, 256),
])
def test_varlen_matches_oracle_per_sequence(lengths, d, R):
    from mamba_selective_scan_jamba_b200 import jmix
    base = synth.Workload("varlen", 1, 1, d, R, "bf16", seed=21, extra=True)
    W, per, x, z, ic, iss, cu = _packed_inputs(base, lengths)
    status, y, fs, fc = _run_varlen(base, lengths, x, z, W, ic, iss, cu)
    assert status == jmix.JM_OK, jmix.jm_last_error()
    tol = TOL["bf16"]
    for b, L in enumerate(lengths):
        if L == 0:
            np.testing.assert_array_equal(fs[b], iss[b])
            np.testing.assert_array_equal(fc[b], ic[b])
            continue
        A = per[b]
        m = oracle.dims_of(base, batch=1, seqlen=L)
        mm = oracle.dims_of(base, batch=1, seqlen=L, mirror=True)
        yr, _, fcr = oracle.mixer_fwd(m, A["x"], A["z"], W, A["init_conv_state"],
                                      A["init_ssm_state"])
        _, fsm, _ = oracle.mixer_fwd(mm, A["x"], A["z"], W, A["init_conv_state"],
                                     A["init_ssm_state"])
        yg = f64(y[cu[b]:cu[b + 1]])
        assert max_scaled_err(yg, yr[0]) <= tol["y"], (b, L)
        assert max_scaled_err(fs[b], fsm[0]) <= tol["state"], (b, L)
        np.testing.assert_array_equal(f64(fc[b]), fcr[0])


def test_varlen_equal_lengths_is_the_fixed_forward():
    """With equal lengths (one scan part each) the packed call computes exactly
    what jm_mixer_fwd computes: the same bits."""
    from tests.helpers import gpu_fwd
    from mamba_selective_scan_jamba_b200 import jmix, devio
    w = synth.Workload("eq", 3, 300, 256, 32, "bf16", seed=8, extra=True)
    assert jmix.jm_mixer_fwd_schedule(devio.dims_of(w)) == (1, False)
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    y, fs, fc = gpu_fwd(w, W, A)
    cu = np.arange(0, 4 * 300, 300, dtype=np.int32)
    status, yv, fsv, fcv = _run_varlen(w, [300] * 3, A["x"].reshape(900, 256),
                                       A["z"].reshape(900, 256), W, A["init_conv_state"],
                                       A["init_ssm_state"], cu)
    assert status == jmix.JM_OK
    np.testing.assert_array_equal(yv.reshape(y.shape), y)
    np.testing.assert_array_equal(fsv, fs)
    np.testing.assert_array_equal(fcv, fc)


def test_varlen_reports_broken_offsets():
    """cu_seqlens that does not end at the token count: the call stays inside its
    buffers and jm_poll_error reports JM_ERR_INVALID_ARG."""
    from mamba_selective_scan_jamba_b200 import jmix
    base = synth.Workload("bad", 1, 1, 256, 16, "bf16", seed=3, extra=True)
    lengths = [10, 20]
    W, per, x, z, ic, iss, cu = _packed_inputs(base, lengths)
    bad = cu.copy()
    bad[-1] = 25            # < T = 30
    status, *_ = _run_varlen(base, lengths, x, z, W, ic, iss, bad)
    assert status == jmix.JM_ERR_INVALID_ARG
    assert "cu_seqlens" in jmix.jm_last_error()
    bad = cu.copy()
    bad[1] = 40             # decreasing offsets
    status, *_ = _run_varlen(base, lengths, x, z, W, ic, iss, bad)
    assert status == jmix.JM_ERR_INVALID_ARG

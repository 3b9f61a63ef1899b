"""jm_mixer_step_indexed: decode steps whose rows use slots of a state pool
(continuous batching), with and without prepared fp16 weights, on cuda:0.

Each step's active rows map to distinct, permuted, sparse slots; the set changes
from step to step.  Checked: every active row against the fp64 oracle run on the
gathered states; the same bits as jm_mixer_step on a dense copy of those states;
identical bits in every slot no row used; a slot outside the pool reported by
jm_poll_error with nothing written for that row.
"""
import numpy as np
import pytest

import oracle
from mamba_selective_scan_jamba_b200 import synth
from tests.helpers import TOL, f64, max_scaled_err

pytestmark = pytest.mark.gpu


def _pool(w, S):
    """Seeded conv and SSM state pools of S slots (the decode recipe's values)."""
    S_ = synth.make_decode_state(w.with_(batch=S))
    return S_["conv_state"], S_["ssm_state"]


def _active_sets(S, B, steps, seed):
    r = np.random.default_rng(seed)
    return [r.permutation(S)[:B].astype(np.int32) for _ in range(steps)]


def run_indexed(w, S, steps, prepared, channels=None, seed=5):
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    B = w.batch
    W = synth.make_weights(w)
    Wd = devio.weights_to_device(W)
    cpool_h, spool_h = _pool(w, S)
    cpool, spool = devio.to_device(cpool_h), devio.to_device(spool_h)
    d = devio.dims_of(w)
    n = jmix.jm_mixer_step_workspace_size(d)
    ws = devio.workspace(n)
    prep = None
    if prepared:
        npw = jmix.jm_prepared_weights_size(d)
        prep = devio.workspace(npw)
        jmix.jm_prepare_weights(d, Wd["xproj_w"], Wd["dtproj_w"], prep, npw)
    ch = np.arange(w.d_inner) if channels is None else np.asarray(channels)
    m_ex = oracle.dims_of(w, seqlen=1)
    m_mi = oracle.dims_of(w, seqlen=1, mirror=True)
    ref_c = f64(cpool_h)                       # conv pool: exact copies of inputs
    ref_s_mi = f64(spool_h)                    # SSM pool under the mirror-rounded oracle
    ref_s_ex = f64(spool_h)
    worst = {"y": 0.0, "y_mirror": 0.0}
    for t, idx in enumerate(_active_sets(S, B, steps, seed)):
        tok = synth.make_decode_token(w, t)
        xt, zt = devio.to_device(tok["x_t"]), devio.to_device(tok["z_t"])
        yt = torch.empty_like(xt)
        before_c, before_s = cpool.clone(), spool.clone()
        idx_d = torch.from_numpy(idx).to("cuda")
        jmix.jm_mixer_step_indexed(d, idx_d, S, xt, zt, cpool, spool, Wd, prep, yt, ws, n)
        assert jmix.jm_poll_error(ws) == jmix.JM_OK, jmix.jm_last_error()
        # the same bits as the dense step on a gathered copy of the active slots
        cs_g, ss_g = before_c[idx_d.long()].clone(), before_s[idx_d.long()].clone()
        yd = torch.empty_like(xt)
        jmix.jm_mixer_step(d, xt, zt, cs_g, ss_g, Wd, yd, ws, n)
        torch.cuda.synchronize()
        assert torch.equal(yt, yd)
        assert torch.equal(cpool[idx_d.long()], cs_g) and torch.equal(spool[idx_d.long()], ss_g)
        # slots no row used keep their bits
        untouched = np.setdiff1d(np.arange(S), idx)
        ut = torch.from_numpy(untouched).to("cuda").long()
        assert torch.equal(cpool[ut], before_c[ut]) and torch.equal(spool[ut], before_s[ut])
        # the oracle on the gathered states
        x3, z3 = tok["x_t"][:, None, :], tok["z_t"][:, None, :]
        y_ex, fs_ex, _ = oracle.mixer_fwd(m_ex, x3, z3, W, ref_c[idx], ref_s_ex[idx], channels=ch)
        ym, fs_mi, _ = oracle.mixer_fwd(m_mi, x3, z3, W, ref_c[idx], ref_s_mi[idx], channels=ch)
        for k, sl in enumerate(idx):
            ref_s_ex[sl][ch] = fs_ex[k]
            ref_s_mi[sl][ch] = fs_mi[k]
        ref_c[idx] = np.concatenate([ref_c[idx][:, :, 1:], f64(tok["x_t"])[:, :, None]], axis=2)
        yg = f64(devio.to_host(yt))[:, ch]
        worst["y"] = max(worst["y"], max_scaled_err(yg, y_ex[:, 0]))
        worst["y_mirror"] = max(worst["y_mirror"], max_scaled_err(yg, ym[:, 0]))
    tol = TOL["bf16"]
    worst["state"] = max_scaled_err(devio.to_host(spool)[:, ch], ref_s_mi[:, ch])
    np.testing.assert_array_equal(f64(devio.to_host(cpool)), ref_c)
    assert worst["y"] <= tol["y"] and worst["y_mirror"] <= tol["y_mirror"], worst
    assert worst["state"] <= tol["state"], worst
    return worst


@pytest.mark.parametrize("prepared", [False, True])
def test_indexed_small(prepared):
    # dt_rank 64: one fp16 rounding flip of dt_n moves delta by about 2^-10/sqrt(R)
    # relative; at R = 16 over 12 rows x 4 steps that alone nears the 1e-4 state gate
    w = synth.Workload("idx", 12, 1, 256, 64, "bf16", seed=41, extra=True, steps=4)
    run_indexed(w, 40, 4, prepared)


def test_indexed_full_pool_permuted():
    """Every slot active, in a permuted order (the pool size equals the batch)."""
    w = synth.Workload("idx_full", 20, 1, 384, 32, "bf16", seed=43, extra=True, steps=2)
    run_indexed(w, 20, 2, True, seed=9)


@pytest.mark.slow
def test_indexed_jamba_b256_in_1024_slots():
    w = synth.WORKLOADS["jamba_decode_b256"]
    run_indexed(w, 1024, 3, True, channels=[0, 1, 31, 32, 4095, 4096, 8160, 8191])


def test_prepared_weights_give_the_same_bits_as_converting():
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    w = synth.Workload("idx_prep", 8, 1, 512, 64, "bf16", seed=47, extra=True, steps=1)
    W = synth.make_weights(w)
    Wd = devio.weights_to_device(W)
    c_h, s_h = _pool(w, 8)
    d = devio.dims_of(w)
    n = jmix.jm_mixer_step_workspace_size(d)
    ws = devio.workspace(n)
    npw = jmix.jm_prepared_weights_size(d)
    prep = devio.workspace(npw)
    jmix.jm_prepare_weights(d, Wd["xproj_w"], Wd["dtproj_w"], prep, npw)
    tok = synth.make_decode_token(w, 0)
    xt, zt = devio.to_device(tok["x_t"]), devio.to_device(tok["z_t"])
    idx = torch.arange(8, dtype=torch.int32, device="cuda")
    outs = []
    for p in (None, prep):
        cp, sp = devio.to_device(c_h), devio.to_device(s_h)
        yt = torch.empty_like(xt)
        jmix.jm_mixer_step_indexed(d, idx, 8, xt, zt, cp, sp, Wd, p, yt, ws, n)
        torch.cuda.synchronize()
        outs.append((yt, cp, sp))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_slot_outside_the_pool_is_reported_and_skipped():
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    w = synth.Workload("idx_bad", 4, 1, 256, 16, "bf16", seed=49, extra=True, steps=1)
    W = synth.make_weights(w)
    Wd = devio.weights_to_device(W)
    c_h, s_h = _pool(w, 6)
    cp, sp = devio.to_device(c_h), devio.to_device(s_h)
    c0, s0 = cp.clone(), sp.clone()
    d = devio.dims_of(w)
    n = jmix.jm_mixer_step_workspace_size(d)
    ws = devio.workspace(n)
    tok = synth.make_decode_token(w, 0)
    xt, zt = devio.to_device(tok["x_t"]), devio.to_device(tok["z_t"])
    yt = torch.full_like(xt, 7.0)
    idx = torch.tensor([3, 6, 0, -1], dtype=torch.int32, device="cuda")   # 6 and -1 are outside
    jmix.jm_mixer_step_indexed(d, idx, 6, xt, zt, cp, sp, Wd, None, yt, ws, n)
    assert jmix.jm_poll_error(ws) == jmix.JM_ERR_INVALID_ARG
    assert "state_idx" in jmix.jm_last_error()
    torch.cuda.synchronize()
    assert (yt[1].float() == 7.0).all() and (yt[3].float() == 7.0).all()   # rows left unwritten
    for s in (1, 2, 4, 5):                                                  # slots no row used
        assert torch.equal(cp[s], c0[s]) and torch.equal(sp[s], s0[s])
    assert not torch.equal(sp[3], s0[3]) and not torch.equal(sp[0], s0[0])
    # the rows after a skipped one are computed exactly as when every slot is valid
    cp2, sp2 = devio.to_device(c_h), devio.to_device(s_h)
    yt2 = torch.full_like(xt, 7.0)
    idx2 = torch.tensor([3, 1, 0, 2], dtype=torch.int32, device="cuda")
    jmix.jm_mixer_step_indexed(d, idx2, 6, xt, zt, cp2, sp2, Wd, None, yt2, ws, n)
    assert jmix.jm_poll_error(ws) == jmix.JM_OK, jmix.jm_last_error()
    torch.cuda.synchronize()
    assert torch.equal(yt[0], yt2[0]) and torch.equal(yt[2], yt2[2])
    for s in (3, 0):
        assert torch.equal(cp[s], cp2[s]) and torch.equal(sp[s], sp2[s])

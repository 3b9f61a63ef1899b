"""jm_scan_bwd on cuda:0 against the fp64 oracle's reverse mode (which is pinned
to finite differences of the forward), for every gradient.

float32 on the GPU against float64: each gradient within 1e-4 max(1, |ref|);
the sums (g_A_log, g_D over tokens and sequences; g_B, g_C over channels) are
reduced in a fixed order, so two runs give the same bits.
"""
import numpy as np
import pytest

import oracle
from tests.helpers import max_scaled_err

pytestmark = pytest.mark.gpu


def _inputs(B, L, d, seed, with_h0=True):
    r = np.random.default_rng(seed)
    f = np.float32
    return dict(delta=np.exp(r.uniform(np.log(1e-3), np.log(0.5), size=(B, L, d))).astype(f),
                u=r.normal(size=(B, L, d)).astype(f), Bm=r.normal(size=(B, L, 16)).astype(f),
                Cm=r.normal(size=(B, L, 16)).astype(f),
                A_log=r.uniform(np.log(0.3), np.log(4.0), size=(d, 16)).astype(f),
                D=r.normal(size=d).astype(f),
                h0=r.normal(size=(B, d, 16)).astype(f) if with_h0 else None,
                gy=r.normal(size=(B, L, d)).astype(f))


def _gpu_bwd(p):
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    B, L, d = p["delta"].shape
    T = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    dev = {k: T(v) for k, v in p.items()}
    out = dict(delta=torch.empty((B, L, d), device="cuda"), u=torch.empty((B, L, d), device="cuda"),
               B=torch.empty((B, L, 16), device="cuda"), C=torch.empty((B, L, 16), device="cuda"),
               A_log=torch.empty((d, 16), device="cuda"), D=torch.empty(d, device="cuda"),
               h0=torch.empty((B, d, 16), device="cuda"))
    dm = jmix.dims(B, L, d, 8)
    n = jmix.jm_scan_bwd_workspace_size(dm)
    ws = devio.workspace(n)
    jmix.jm_scan_bwd(dm, dev["delta"], dev["u"], dev["Bm"], dev["Cm"], dev["A_log"], dev["D"],
                     dev["h0"], dev["gy"], out["delta"], out["u"], out["B"], out["C"],
                     out["A_log"], out["D"], out["h0"], ws, n)
    assert jmix.jm_poll_error(ws) == jmix.JM_OK
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def _oracle_bwd(p):
    B = p["delta"].shape[0]
    acc = None
    per = []
    for b in range(B):
        g = oracle.scan_bwd(p["delta"][b], p["A_log"], p["Bm"][b], p["Cm"][b], p["u"][b], p["D"],
                            None if p["h0"] is None else p["h0"][b], p["gy"][b])
        per.append(g)
    return dict(delta=np.stack([g["delta"] for g in per]), u=np.stack([g["u"] for g in per]),
                B=np.stack([g["B"] for g in per]), C=np.stack([g["C"] for g in per]),
                A_log=sum(g["A_log"] for g in per), D=sum(g["D"] for g in per),
                h0=np.stack([g["h0"] for g in per]))


# (2, 301, 384) and (1, 1000, 1024) run as 16 time parts (ragged parts and a
# ragged last chunk); (2, 37, 200) and (3, 4, 128) as one part.
@pytest.mark.parametrize("B,L,d,h0", [(2, 37, 200, True), (1, 1000, 1024, False),
                                      (3, 4, 128, True), (2, 301, 384, True),
                                      (1, 2048, 2048, True)])
def test_scan_bwd_matches_oracle(B, L, d, h0):
    p = _inputs(B, L, d, seed=B * 1000 + L, with_h0=h0)
    got = _gpu_bwd(p)
    ref = _oracle_bwd(p)
    for k in ref:
        assert max_scaled_err(got[k], ref[k]) <= 1e-4, (k, max_scaled_err(got[k], ref[k]))
    again = _gpu_bwd(p)
    for k in got:
        np.testing.assert_array_equal(again[k], got[k])


def test_scan_bwd_empty_sequence():
    p = _inputs(2, 0, 128, seed=5)
    got = _gpu_bwd(p)
    assert not got["A_log"].any() and not got["D"].any() and not got["h0"].any()

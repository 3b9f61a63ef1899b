"""Pins of the fp64 oracle to facts other than itself (CPU only).

The pages print no worked numbers for the mixer, so each part of the oracle is
tied to a closed form, a brute-force restatement, an invariant or a textbook
identity, each chosen so that a plausible mistake (a dropped term, a wrong
sign, an off-by-one in time, B and C swapped, the conv taps reversed, eps
outside the root) fails at least one test.  The tests call only ``oracle``
and the seeded input generator.
"""
import math

import numpy as np
import pytest

import oracle
from mamba_selective_scan_jamba_b200 import synth

RNG = np.random.default_rng(20240328)


def rand_scan_inputs(L, d, N, with_h0=True, seed=0):
    r = np.random.default_rng(seed)
    delta = np.exp(r.uniform(np.log(1e-3), np.log(0.5), size=(L, d)))
    A = -np.exp(r.uniform(np.log(0.25), np.log(8.0), size=(d, N)))
    Bm = r.normal(size=(L, N))
    Cm = r.normal(size=(L, N))
    u = r.normal(size=(L, d))
    D = r.normal(size=d)
    h0 = r.normal(size=(d, N)) if with_h0 else None
    return delta, A, Bm, Cm, u, D, h0


# ------------------------------------------------------------------ scan core
def test_scan_L1_closed_form():
    """L = 1 from h0 = 0: h = delta*B*u and y = C.(delta*B*u) + D*u."""
    delta, A, Bm, Cm, u, D, _ = rand_scan_inputs(1, 5, 16, seed=1)
    y, hT = oracle.scan(delta, A, Bm, Cm, u, D, None)
    h = delta[0][:, None] * Bm[0][None, :] * u[0][:, None]
    np.testing.assert_allclose(hT, h, rtol=1e-14, atol=0)
    np.testing.assert_allclose(y[0], h @ Cm[0] + D * u[0], rtol=1e-14, atol=1e-15)


def test_scan_geometric_series():
    """Constant delta, A, B, C, u: h_t = a^t h0 + b (1 - a^t) / (1 - a), a = exp(delta A),
    b = delta B u, with t counting updates (h_1 is the state after the first token)."""
    L, d, N = 37, 3, 16
    r = np.random.default_rng(2)
    dl = np.array([0.01, 0.3, 2.0])
    A = -np.exp(r.uniform(-1, 2, size=(d, N)))
    B1, C1 = r.normal(size=N), r.normal(size=N)
    u1 = np.array([0.7, -1.3, 0.2])
    D = r.normal(size=d)
    h0 = r.normal(size=(d, N))
    delta = np.tile(dl, (L, 1))
    y, hT = oracle.scan(delta, A, np.tile(B1, (L, 1)), np.tile(C1, (L, 1)), np.tile(u1, (L, 1)),
                        D, h0)
    a = np.exp(dl[:, None] * A)
    b = dl[:, None] * B1[None, :] * u1[:, None]
    for t in (1, 2, 10, L):
        ht = a ** t * h0 + b * (1 - a ** t) / (1 - a)
        np.testing.assert_allclose(y[t - 1], ht @ C1 + D * u1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(hT, a ** L * h0 + b * (1 - a ** L) / (1 - a), rtol=1e-12, atol=1e-14)


def hidden_attention(delta, A, Bm, Cm, u, D, h0):
    """Materialised form (Ali, Zimerman & Wolf, "The hidden attention of Mamba
    models", cited by the Jamba paper): y_t = sum_{s<=t} sum_n C_t,n
    (prod_{r=s+1..t} e^{delta_r A_n}) delta_s B_s,n u_s + C_t.(prod_{r<=t} e^{delta_r A}) h0
    + D u_t, one term at a time."""
    L, d = delta.shape
    N = A.shape[1]
    y = np.zeros((L, d))
    for c in range(d):
        for t in range(L):
            acc = 0.0
            for n in range(N):
                for s in range(t + 1):
                    decay = 1.0
                    for rr in range(s + 1, t + 1):
                        decay *= math.exp(delta[rr, c] * A[c, n])
                    acc += Cm[t, n] * decay * delta[s, c] * Bm[s, n] * u[s, c]
                if h0 is not None:
                    decay = 1.0
                    for rr in range(0, t + 1):
                        decay *= math.exp(delta[rr, c] * A[c, n])
                    acc += Cm[t, n] * decay * h0[c, n]
            y[t, c] = acc + D[c] * u[t, c]
    return y


@pytest.mark.parametrize("L,d,N,with_h0", [(1, 2, 3, False), (7, 3, 4, True), (13, 2, 16, True)])
def test_scan_hidden_attention_bruteforce(L, d, N, with_h0):
    delta, A, Bm, Cm, u, D, h0 = rand_scan_inputs(L, d, N, with_h0, seed=L * 31 + d)
    y, _ = oracle.scan(delta, A, Bm, Cm, u, D, h0)
    np.testing.assert_allclose(y, hidden_attention(delta, A, Bm, Cm, u, D, h0), rtol=1e-12,
                               atol=1e-13)


def test_scan_matches_guide_toy_loop():
    """The aifetchly guide's toy SSM (``SimpleMambaSSM.forward``) discretises with
    exp(delta A) and delta B, zero initial state, no D: vectorised over channels
    here, one time step per iteration."""
    L, d, N = 9, 4, 16
    delta, A, Bm, Cm, u, _, _ = rand_scan_inputs(L, d, N, seed=5)
    dA = np.exp(delta[:, :, None] * A[None, :, :])           # [L, d, N]
    dB = delta[:, :, None] * Bm[:, None, :]                   # [L, d, N]
    h = np.zeros((d, N))
    ys = []
    for t in range(L):
        h = dA[t] * h + dB[t] * u[t][:, None]
        ys.append((h * Cm[t][None, :]).sum(-1))
    y, _ = oracle.scan(delta, A, Bm, Cm, u, np.zeros(d), None)
    np.testing.assert_allclose(y, np.stack(ys), rtol=1e-13, atol=1e-14)


def test_scan_limits_and_linearity():
    L, d, N = 11, 3, 16
    delta, A, Bm, Cm, u, D, h0 = rand_scan_inputs(L, d, N, seed=6)
    # delta -> 0: the state never moves; y = C_t.h0 + D u_t
    y, hT = oracle.scan(np.zeros_like(delta), A, Bm, Cm, u, D, h0)
    np.testing.assert_allclose(hT, h0, rtol=0, atol=0)
    np.testing.assert_allclose(y, Cm @ h0.T + D * u, rtol=1e-13, atol=1e-14)
    # very fast decay: the state forgets everything but the current token
    big = np.full_like(delta, 1.0)
    Abig = np.full_like(A, -1e4)
    y, hT = oracle.scan(big, Abig, Bm, Cm, u, D, h0)
    np.testing.assert_allclose(hT, (Bm[-1][None, :] * u[-1][:, None]), rtol=1e-12)
    # linearity in (u, h0) for fixed delta, A, B, C, D
    u2 = np.random.default_rng(7).normal(size=u.shape)
    h02 = np.random.default_rng(8).normal(size=h0.shape)
    ya, ha = oracle.scan(delta, A, Bm, Cm, u, D, h0)
    yb, hb = oracle.scan(delta, A, Bm, Cm, u2, D, h02)
    yc, hc = oracle.scan(delta, A, Bm, Cm, 2 * u - 3 * u2, D, 2 * h0 - 3 * h02)
    np.testing.assert_allclose(yc, 2 * ya - 3 * yb, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(hc, 2 * ha - 3 * hb, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------- front-end pieces
def test_conv_impulse_response_and_history():
    """A unit impulse at t = 0 returns the taps reversed in time: the last tap
    multiplies the current token.  With x = 0, only the cached history acts."""
    L, d, K = 6, 3, 4
    r = np.random.default_rng(9)
    w = r.normal(size=(d, K))
    b = r.normal(size=d)
    x = np.zeros((L, d))
    x[0, :] = 1.0
    xc = oracle.conv(x, w, b)
    for t in range(L):
        want = b + (w[:, K - 1 - t] if t < K else 0.0)
        np.testing.assert_array_equal(xc[t], want)
    hist = r.normal(size=(d, K - 1))   # oldest first
    xc = oracle.conv(np.zeros((L, d)), w, np.zeros(d), hist)
    np.testing.assert_allclose(xc[0], (w[:, :K - 1] * hist).sum(1), rtol=1e-15)
    np.testing.assert_allclose(xc[1], (w[:, :K - 2] * hist[:, 1:]).sum(1), rtol=1e-15)
    np.testing.assert_allclose(xc[2], w[:, 0] * hist[:, 2], rtol=1e-15)
    np.testing.assert_array_equal(xc[3:], 0.0)


def test_silu_identities():
    v = np.linspace(-30, 30, 1201)
    s = oracle.silu(v)
    np.testing.assert_allclose(s - oracle.silu(-v), v, rtol=1e-14, atol=1e-14)  # x(s(x)+s(-x)) = x
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(oracle.silu(np.array([40.0])), [40.0], rtol=1e-15)


def test_rmsnorm_identities():
    r = np.random.default_rng(10)
    v = r.normal(size=(5, 256)) * 3.0
    out = oracle.rmsnorm(v, np.ones(256), 0.0)
    np.testing.assert_allclose(np.sqrt((out ** 2).mean(-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(oracle.rmsnorm(7.5 * v, np.ones(256), 0.0), out, rtol=1e-14)
    # eps sits inside the root: a constant vector a*1 maps to a / sqrt(a^2 + eps)
    a, eps = 0.01, 1e-6
    np.testing.assert_allclose(oracle.rmsnorm(np.full((1, 16), a), np.ones(16), eps),
                               np.full((1, 16), a / math.sqrt(a * a + eps)), rtol=1e-15)
    w = r.normal(size=16)
    np.testing.assert_allclose(oracle.rmsnorm(v[:, :16], w, 0.0),
                               oracle.rmsnorm(v[:, :16], np.ones(16), 0.0) * w, rtol=1e-15)


def test_softplus_identities():
    dt = np.exp(np.linspace(np.log(1e-6), np.log(50.0), 500))
    inv = np.log(np.expm1(dt))   # softplus^-1
    np.testing.assert_allclose(oracle.softplus(inv), dt, rtol=1e-13)
    assert abs(oracle.softplus1(0.0) - math.log(2.0)) < 1e-16
    assert abs(oracle.softplus1(-40.0) - math.exp(-40.0)) < 1e-30
    assert oracle.softplus1(800.0) == 800.0


def test_round_fp16():
    assert oracle.round_fp16(1.0) == 1.0
    assert oracle.round_fp16(1.0 + 2 ** -11) == 1.0                   # tie -> even
    assert oracle.round_fp16(1.0 + 3 * 2 ** -11) == 1.0 + 2 ** -9     # tie -> even (up)
    assert oracle.round_fp16(2 ** -24) == 2 ** -24                    # smallest subnormal kept
    assert oracle.round_fp16(65504.0) == 65504.0
    np.testing.assert_equal(np.float16(0.1).astype(np.float64), oracle.round_fp16(0.1))


def test_round_bf16():
    assert oracle.round_bf16(1.0) == 1.0
    assert oracle.round_bf16(1.0 + 2 ** -8) == 1.0            # tie -> even
    assert oracle.round_bf16(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6  # tie -> even (up)
    assert oracle.round_bf16(1.0 + 2 ** -8 + 2 ** -20) == 1.0 + 2 ** -7


# ------------------------------------------------------------- whole mixer
def tiny(extra=True, io="f32", L=24, d=40, R=8, B=2, seed=11):
    return synth.Workload("pin", B, L, d, R, io, seed=seed, extra=extra)


def test_mixer_split_invariant():
    """Running [0, L1) and then [L1, L) from the carried conv and SSM states
    reproduces the full run, including cuts inside the conv window."""
    w = tiny()
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    m = oracle.dims_of(w)
    y, fs, fc = oracle.mixer_fwd(m, A["x"], A["z"], W, A["init_conv_state"], A["init_ssm_state"])
    for L1 in (1, 2, 3, 17):
        m1 = oracle.dims_of(w, seqlen=L1)
        m2 = oracle.dims_of(w, seqlen=w.seqlen - L1)
        y1, s1, c1 = oracle.mixer_fwd(m1, A["x"][:, :L1], A["z"][:, :L1], W, A["init_conv_state"],
                                      A["init_ssm_state"])
        y2, s2, c2 = oracle.mixer_fwd(m2, A["x"][:, L1:], A["z"][:, L1:], W, c1, s1)
        np.testing.assert_allclose(np.concatenate([y1, y2], 1), y, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(s2, fs, rtol=1e-12, atol=1e-13)
        np.testing.assert_array_equal(c2, fc)


def test_mixer_step_equals_forward():
    w = tiny(L=9)
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    m = oracle.dims_of(w)
    y, fs, fc = oracle.mixer_fwd(m, A["x"], A["z"], W, A["init_conv_state"], A["init_ssm_state"])
    cs, ss = A["init_conv_state"], A["init_ssm_state"]
    ms = oracle.dims_of(w, seqlen=1)
    for t in range(w.seqlen):
        yt, cs, ss = oracle.mixer_step(ms, A["x"][:, t], A["z"][:, t], cs, ss, W)
        np.testing.assert_allclose(yt, y[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ss, fs, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(cs, fc)


def test_mixer_channel_permutation_and_batch_independence():
    w = tiny(B=3)
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    m = oracle.dims_of(w)
    y, fs, fc = oracle.mixer_fwd(m, A["x"], A["z"], W, A["init_conv_state"], A["init_ssm_state"])
    perm = np.random.default_rng(12).permutation(w.d_inner)
    Wp = dict(W)
    for k in ("conv_w", "conv_b", "dtproj_w", "dt_bias", "A_log", "D"):
        Wp[k] = W[k][perm]
    Wp["xproj_w"] = W["xproj_w"][:, perm]
    yp, fsp, fcp = oracle.mixer_fwd(m, A["x"][:, :, perm], A["z"][:, :, perm], Wp,
                                    A["init_conv_state"][:, perm], A["init_ssm_state"][:, perm])
    np.testing.assert_allclose(yp, y[:, :, perm], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(fsp, fs[:, perm], rtol=1e-13, atol=1e-14)
    m1 = oracle.dims_of(w, batch=1)
    for b in range(w.batch):
        yb, fsb, _ = oracle.mixer_fwd(m1, A["x"][b:b + 1], A["z"][b:b + 1], W,
                                      A["init_conv_state"][b:b + 1], A["init_ssm_state"][b:b + 1])
        np.testing.assert_array_equal(yb[0], y[b])
        np.testing.assert_array_equal(fsb[0], fs[b])


def test_mixer_gate_skip_and_split_order():
    """x_proj rows are [dt | B | C].  With the C rows zeroed the output is the
    skip path alone, y = D u SiLU(z); with the B rows zeroed and h0 = 0 the
    state never leaves zero; with the dt rows zeroed, delta = softplus(dt_bias)."""
    w = tiny(extra=True, B=1)
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    R, N = w.dt_rank, w.d_state
    m = oracle.dims_of(w)
    x = A["x"][0].astype(np.float64)
    u = oracle.silu(oracle.conv(x, W["conv_w"], W["conv_b"], A["init_conv_state"][0]))
    gate = oracle.silu(A["z"][0])
    # C rows zero
    Wc = dict(W)
    Wc["xproj_w"] = W["xproj_w"].copy()
    Wc["xproj_w"][R + N:] = 0
    y, fs, _ = oracle.mixer_fwd(m, A["x"], A["z"], Wc, A["init_conv_state"], None)
    np.testing.assert_allclose(y[0], W["D"] * u * gate, rtol=1e-13, atol=1e-14)
    assert np.abs(fs).max() > 0
    # B rows zero, h0 = 0: state stays 0, y = D u SiLU(z)
    Wb = dict(W)
    Wb["xproj_w"] = W["xproj_w"].copy()
    Wb["xproj_w"][R:R + N] = 0
    y, fs, _ = oracle.mixer_fwd(m, A["x"], A["z"], Wb, A["init_conv_state"], None)
    np.testing.assert_array_equal(fs, 0.0)
    np.testing.assert_allclose(y[0], W["D"] * u * gate, rtol=1e-13, atol=1e-14)
    # dt rows zero: delta = softplus(dt_bias) for every token
    Wd = dict(W)
    Wd["xproj_w"] = W["xproj_w"].copy()
    Wd["xproj_w"][:R] = 0
    y, fs, _ = oracle.mixer_fwd(m, A["x"], A["z"], Wd, A["init_conv_state"], A["init_ssm_state"])
    p = u @ W["xproj_w"].astype(np.float64).T
    Bn = oracle.rmsnorm(p[:, R:R + N], W["b_norm_w"], w.eps)
    Cn = oracle.rmsnorm(p[:, R + N:], W["c_norm_w"], w.eps)
    delta = np.tile(np.log1p(np.exp(W["dt_bias"].astype(np.float64))), (w.seqlen, 1))
    ys, hT = oracle.scan(delta, -np.exp(W["A_log"].astype(np.float64)), Bn, Cn, u, W["D"],
                         A["init_ssm_state"][0])
    np.testing.assert_allclose(y[0], ys * gate, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fs[0], hT, rtol=1e-11, atol=1e-13)


# ------------------------------------------------------------- the dt branch
# delta = softplus(W_dt . (RMSNorm(dt) w_dt) + dt_bias), with dt the first R
# outputs of x_proj (TransformerLens "Jamba" adapter page, "Key adapter
# decisions": the three RMSNorms on the selective parameters, applied before
# dt_proj; aifetchly "Jamba Guide", "Hands-On Implementation": delta =
# softplus(dt_proj(.))).  Each check raises AssertionError when it fails; the
# planted-mistake tests (test_oracle_planted.py) run the same checks on
# mutated copies of the oracle.

def _dt_case(seed=21):
    w = synth.Workload("dtpin", 2, 13, 40, 8, "f32", seed=seed, extra=True)
    W = {k: np.asarray(v, dtype=np.float64) for k, v in synth.make_weights(w).items()}
    return w, W, synth.make_activations(w)


def _dt_run(w, W, A, eps):
    m = oracle.dims(w.batch, w.seqlen, w.d_inner, w.dt_rank, eps=eps)
    y, fs, _ = oracle.mixer_fwd(m, A["x"], A["z"], W, A["init_conv_state"], A["init_ssm_state"])
    return y, fs


def _with_dt_rows_scaled(W, R, alpha):
    xw = W["xproj_w"].copy()
    xw[:R] *= alpha
    return dict(W, xproj_w=xw)


def check_dt_rmsnorm_scale_invariance():
    """With eps = 0, RMSNorm(alpha v) = RMSNorm(v) for alpha > 0, so scaling the
    dt rows of xproj_w leaves y and the final state unchanged; alpha = -1 equals
    negating dt_norm_w (the norm is odd in v, and w multiplies after it)."""
    w, W, A = _dt_case()
    R = w.dt_rank
    y, fs = _dt_run(w, W, A, 0.0)
    for alpha in (3.7, 0.21):
        ys, fss = _dt_run(w, _with_dt_rows_scaled(W, R, alpha), A, 0.0)
        np.testing.assert_allclose(ys, y, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(fss, fs, rtol=1e-11, atol=1e-12)
    yn, fsn = _dt_run(w, _with_dt_rows_scaled(W, R, -1.0), A, 0.0)
    ym, fsm = _dt_run(w, dict(W, dt_norm_w=-W["dt_norm_w"]), A, 0.0)
    np.testing.assert_allclose(yn, ym, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(fsn, fsm, rtol=1e-13, atol=1e-14)
    assert np.abs(ym - y).max() > 1e-3      # the dt branch reaches y


def check_dt_norm_weight_equals_dtproj_scaling():
    """dt_proj is linear after the norm's weight: scaling dt_norm_w by alpha equals
    scaling dtproj_w by alpha (any eps, any sign of alpha)."""
    w, W, A = _dt_case()
    y0, _ = _dt_run(w, W, A, w.eps)
    for alpha in (2.5, -0.6):
        y1, fs1 = _dt_run(w, dict(W, dt_norm_w=alpha * W["dt_norm_w"]), A, w.eps)
        y2, fs2 = _dt_run(w, dict(W, dtproj_w=alpha * W["dtproj_w"]), A, w.eps)
        np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(fs1, fs2, rtol=1e-12, atol=1e-13)
        assert np.abs(y1 - y0).max() > 1e-3


def check_dt_onehot_selection():
    """With one-hot dtproj_w rows (channel c reads dt coordinate r(c) alone) the
    contraction is a selection: delta[t, c] = softplus(dt_n[t, r(c)] + dt_bias[c]),
    dt_n = RMSNorm over the R dt outputs with dt_norm_w.  y and the final state
    then equal the separately pinned scan core fed with that delta."""
    w, W, A = _dt_case()
    d, R, N = w.d_inner, w.dt_rank, w.d_state
    r_of_c = (3 * np.arange(d) + 1) % R
    onehot = np.zeros((d, R))
    onehot[np.arange(d), r_of_c] = 1.0
    y, fs = _dt_run(w, dict(W, dtproj_w=onehot), A, w.eps)
    Aneg = -np.exp(W["A_log"])
    for b in range(w.batch):
        u = oracle.silu(oracle.conv(A["x"][b].astype(np.float64), W["conv_w"], W["conv_b"],
                                    A["init_conv_state"][b]))
        p = u @ W["xproj_w"].T
        dtn = oracle.rmsnorm(p[:, :R], W["dt_norm_w"], w.eps)
        Bn = oracle.rmsnorm(p[:, R:R + N], W["b_norm_w"], w.eps)
        Cn = oracle.rmsnorm(p[:, R + N:], W["c_norm_w"], w.eps)
        delta = oracle.softplus(dtn[:, r_of_c] + W["dt_bias"][None, :])
        ys, hT = oracle.scan(delta, Aneg, Bn, Cn, u, W["D"], A["init_ssm_state"][b])
        np.testing.assert_allclose(y[b], ys * oracle.silu(A["z"][b]), rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(fs[b], hT, rtol=1e-11, atol=1e-12)


DT_BRANCH_CHECKS = (check_dt_rmsnorm_scale_invariance, check_dt_norm_weight_equals_dtproj_scaling,
                    check_dt_onehot_selection)


@pytest.mark.parametrize("check", DT_BRANCH_CHECKS, ids=lambda f: f.__name__)
def test_dt_branch(check):
    check()


def test_mirror_rounding_is_small():
    """Mirror mode rounds u and dt_n to fp16; on bf16 inputs it must stay well
    inside the bf16-io output tolerance of the exact run."""
    w = tiny(io="bf16")
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    y, fs, _ = oracle.mixer_fwd(oracle.dims_of(w), A["x"], A["z"], W, A["init_conv_state"],
                                A["init_ssm_state"])
    ym, fsm, _ = oracle.mixer_fwd(oracle.dims_of(w, mirror=True), A["x"], A["z"], W,
                                  A["init_conv_state"], A["init_ssm_state"])
    assert (np.abs(ym - y) / np.maximum(1.0, np.abs(y))).max() < 5e-3
    assert 0 < np.abs(fsm - fs).max() < 2e-3


def test_sampled_channels_match_full():
    w = tiny()
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    m = oracle.dims_of(w)
    y, fs, fc = oracle.mixer_fwd(m, A["x"], A["z"], W, A["init_conv_state"], A["init_ssm_state"])
    ch = [0, 7, 39]
    ys, fss, fcs = oracle.mixer_fwd(m, A["x"], A["z"], W, A["init_conv_state"],
                                    A["init_ssm_state"], channels=ch)
    np.testing.assert_array_equal(ys, y[:, :, ch])
    np.testing.assert_array_equal(fss, fs[:, ch])
    np.testing.assert_array_equal(fcs, fc[:, ch])


# -------------------------------------------------- zero-order-hold variant
def _rk4_step(a, b, h, dt, steps):
    """Integrate dh/dt = a h + b from h over dt by classic Runge-Kutta (RK4)."""
    s = dt / steps
    for _ in range(steps):
        k1 = a * h + b
        k2 = a * (h + 0.5 * s * k1) + b
        k3 = a * (h + 0.5 * s * k2) + b
        k4 = a * (h + s * k3) + b
        h = h + s / 6.0 * (k1 + 2 * k2 + 2 * k3 + k4)
    return h


def test_zoh_step_is_the_exact_ode_step():
    """Zero-order hold is the exact solution of dh/dt = A h + B u over one step with
    u held: the oracle's state after each token matches a fine RK4 integration of
    that ODE (token by token, from the previous state)."""
    L, d, N = 6, 2, 16
    delta, A, Bm, Cm, u, D, h0 = rand_scan_inputs(L, d, N, seed=41)
    h = h0.copy()
    for t in range(L):
        _, hT = oracle.scan(delta[: t + 1], A, Bm[: t + 1], Cm[: t + 1], u[: t + 1], D, h0,
                            zoh=True)
        b = Bm[t][None, :] * u[t][:, None]
        h = _rk4_step(A, b, h, delta[t][:, None], 2000)
        np.testing.assert_allclose(hT, h, rtol=1e-9, atol=1e-11)


def test_zoh_constant_inputs_closed_form():
    """Constant inputs: h_t = a^t h0 + (1 - a^t) h*, with a = exp(delta A) and the
    fixed point h* = -B u / A of dh/dt = A h + B u (no delta in it)."""
    L, d, N = 25, 3, 16
    r = np.random.default_rng(5)
    dl = np.array([0.02, 0.4, 3.0])
    A = -np.exp(r.uniform(-1, 2, size=(d, N)))
    B1, C1 = r.normal(size=N), r.normal(size=N)
    u1 = np.array([0.5, -2.0, 1.1])
    D = r.normal(size=d)
    h0 = r.normal(size=(d, N))
    y, hT = oracle.scan(np.tile(dl, (L, 1)), A, np.tile(B1, (L, 1)), np.tile(C1, (L, 1)),
                        np.tile(u1, (L, 1)), D, h0, zoh=True)
    a = np.exp(dl[:, None] * A)
    hstar = -B1[None, :] * u1[:, None] / A
    for t in (1, 3, L):
        ht = a ** t * h0 + (1 - a ** t) * hstar
        np.testing.assert_allclose(y[t - 1], ht @ C1 + D * u1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hT, a ** L * h0 + (1 - a ** L) * hstar, rtol=1e-12, atol=1e-13)


def test_zoh_L1_and_small_delta_limit():
    """L = 1 from zero: h = (exp(delta A) - 1) / A B u; as delta -> 0 the hold
    and Euler updates agree to first order (difference O(delta^2))."""
    delta, A, Bm, Cm, u, D, _ = rand_scan_inputs(1, 4, 16, seed=7)
    _, hT = oracle.scan(delta, A, Bm, Cm, u, D, None, zoh=True)
    h = np.expm1(delta[0][:, None] * A) / A * Bm[0][None, :] * u[0][:, None]
    np.testing.assert_allclose(hT, h, rtol=1e-14, atol=0)
    for scale in (1e-3, 1e-5):
        dl = delta * scale
        _, hz = oracle.scan(dl, A, Bm, Cm, u, D, None, zoh=True)
        _, he = oracle.scan(dl, A, Bm, Cm, u, D, None)
        rel = np.abs(hz - he).max() / np.abs(he).max()
        assert rel <= 5 * scale * np.abs(A).max() * delta.max(), (scale, rel)
        assert rel > 0


def test_zoh_mixer_wiring():
    """Whole mixer: the flag reaches the scan (results differ at the workloads' delta),
    and with delta driven to ~1e-6 by dt_bias the hold and Euler mixers agree to
    O(delta^2) relative, as they must; a wrong hold factor (a dropped 1/A, a sign)
    fails this at O(1)."""
    w = synth.Workload("zoh", 1, 9, 32, 8, "f32", seed=13, extra=True)
    W = synth.make_weights(w)
    A_ = synth.make_activations(w)
    args = (A_["x"], A_["z"])
    kw = dict(init_conv_state=A_["init_conv_state"])
    ye, _, _ = oracle.mixer_fwd(oracle.dims_of(w), *args, W, **kw)
    yz, _, _ = oracle.mixer_fwd(oracle.dims_of(w, zoh=True), *args, W, **kw)
    assert np.abs(yz - ye).max() > 1e-4
    Wsmall = dict(W, dt_bias=np.full_like(W["dt_bias"], -14.0))   # delta ~ 1e-6 (x O(1))
    ye, fse, _ = oracle.mixer_fwd(oracle.dims_of(w), *args, Wsmall, **kw)
    yz, fsz, _ = oracle.mixer_fwd(oracle.dims_of(w, zoh=True), *args, Wsmall, **kw)
    rel = np.abs(fsz - fse).max() / np.abs(fse).max()
    assert 0 < rel < 1e-4, rel


def test_layer_oracle_with_identity_projections_is_the_mixer():
    """The layer's projections: with d_model = d_inner, in_proj_w = [I; s I] and
    out_proj_w = I, the layer is the mixer on (hidden, s * hidden).  Fixes the x / z
    split order (x first) and the transposes of both products."""
    w = synth.Workload("lay", 2, 11, 24, 8, "f32", seed=17, extra=True)
    W = synth.make_weights(w)
    hidden = np.random.default_rng(3).normal(size=(2, 11, 24))
    s = -0.75
    eye = np.eye(24)
    out, fs = oracle.layer_fwd(oracle.dims_of(w), hidden, np.vstack([eye, s * eye]), eye, W)
    y, fsm, _ = oracle.mixer_fwd(oracle.dims_of(w), hidden, s * hidden, W)
    np.testing.assert_allclose(out, y, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(fs, fsm, rtol=1e-13, atol=1e-14)


# ------------------------------------------------------ backward of the scan
def _loss(delta, A_log, Bm, Cm, u, D, h0, gy):
    """A scalar of the scan core's outputs: <gy, y_s> (its gradient is what
    scan_bwd returns)."""
    y, _ = oracle.scan(delta, -np.exp(A_log), Bm, Cm, u, D, h0)
    return float((gy * y).sum())


def _bwd_inputs(seed, L=7, d=3, N=16):
    r = np.random.default_rng(seed)
    return dict(delta=np.exp(r.uniform(np.log(0.01), np.log(0.8), size=(L, d))),
                A_log=r.uniform(np.log(0.3), np.log(4.0), size=(d, N)),
                Bm=r.normal(size=(L, N)), Cm=r.normal(size=(L, N)), u=r.normal(size=(L, d)),
                D=r.normal(size=d), h0=r.normal(size=(d, N)), gy=r.normal(size=(L, d)))


def test_scan_bwd_matches_central_finite_differences():
    """Every gradient against (f(x + e) - f(x - e)) / 2e of the forward oracle,
    entry by entry, for a few entries of each input (fp64, e = 1e-6)."""
    p = _bwd_inputs(31)
    g = oracle.scan_bwd(p["delta"], p["A_log"], p["Bm"], p["Cm"], p["u"], p["D"], p["h0"],
                        p["gy"])
    names = {"delta": "delta", "A_log": "A_log", "Bm": "B", "Cm": "C", "u": "u", "D": "D",
             "h0": "h0"}
    r = np.random.default_rng(0)
    for key, gname in names.items():
        for _ in range(4):
            idx = tuple(int(r.integers(0, s)) for s in p[key].shape)
            e = 1e-6
            plus = {k: v.copy() for k, v in p.items()}
            minus = {k: v.copy() for k, v in p.items()}
            plus[key][idx] += e
            minus[key][idx] -= e
            fd = (_loss(**plus) - _loss(**minus)) / (2 * e)
            assert abs(g[gname][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (key, idx, g[gname][idx], fd)


def test_scan_bwd_adjoint_dot_product():
    """Linearity in gy: the gradient of <gy1 + 2 gy2, y> is g(gy1) + 2 g(gy2), and
    <g_u(gy), du> equals the directional derivative of <gy, y> along du (the
    forward is linear in h0 and in u for fixed delta, B, C)."""
    p = _bwd_inputs(32)
    r = np.random.default_rng(1)
    gy2 = r.normal(size=p["gy"].shape)
    g1 = oracle.scan_bwd(**{k: v for k, v in p.items()})
    g2 = oracle.scan_bwd(**dict(p, gy=gy2))
    g12 = oracle.scan_bwd(**dict(p, gy=p["gy"] + 2 * gy2))
    for k in g1:
        np.testing.assert_allclose(g12[k], g1[k] + 2 * g2[k], rtol=1e-11, atol=1e-12)
    du, dh0 = r.normal(size=p["u"].shape), r.normal(size=p["h0"].shape)
    base = _loss(**p)
    lin = _loss(**dict(p, u=p["u"] + du, h0=p["h0"] + dh0)) - base
    np.testing.assert_allclose((g1["u"] * du).sum() + (g1["h0"] * dh0).sum(), lin, rtol=1e-11)

"""CPU checks of the C ABI: the library loads, exports every declared entry
point, and rejects bad arguments on the host before any launch (none of the
calls below reaches a CUDA call, so no GPU is needed)."""
import ctypes
import os
import re

import pytest

from mamba_selective_scan_jamba_b200 import build, jmix

HEADER = os.path.join(build.INCLUDE, "jmix.h")


@pytest.fixture(scope="module")
def lib():
    build.build_libjmix()
    return jmix.load()


def declared_entry_points():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(jm_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_entry_points()
    assert "jm_mixer_fwd" in names and "jm_mixer_step" in names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(jmix.EXPORTED) == names


def test_no_other_symbols_exported():
    out = os.popen(f"nm -D --defined-only {jmix.LIB_PATH}").read()
    syms = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert sorted(syms) == sorted(jmix.EXPORTED)


def test_built_for_sm100a_only():
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1


FAKE = 1 << 40   # an aligned, never-dereferenced address


def fwd(d, ws_bytes=1 << 30, **over):
    args = dict(x=FAKE, z=FAKE + (1 << 36), y=FAKE + (2 << 36), final_state=FAKE,
                workspace=FAKE, init_conv_state=None, init_ssm_state=None, final_conv_state=None)
    args.update(over)
    W = {k: FAKE for k in jmix.WEIGHT_NAMES}
    return jmix.jm_mixer_fwd(d, args["x"], args["z"], W, args["y"], args["final_state"],
                             args["workspace"], ws_bytes, args["init_conv_state"],
                             args["init_ssm_state"], args["final_conv_state"], stream=0,
                             check=False)


def test_workspace_size_of_empty_problems(lib):
    for io in (jmix.JM_BF16, jmix.JM_F32):
        for B, L in ((0, 5), (2, 0), (0, 0)):
            assert jmix.jm_mixer_fwd_workspace_size(jmix.dims(B, L, 256, 16, io)) >= 256
        assert jmix.jm_mixer_step_workspace_size(jmix.dims(0, 1, 256, 16, io)) >= 256


def test_workspace_size_rules(lib):
    d = jmix.dims(8, 4096, 8192, 256)
    n = jmix.jm_mixer_fwd_workspace_size(d)
    assert n >= 256 + 8 * 4096 * 288 * 4
    assert jmix.jm_mixer_fwd_workspace_size(jmix.dims(1, 4096, 8192, 256, d_state=8)) == 0
    assert "d_state" in jmix.jm_last_error()
    assert jmix.jm_mixer_step_workspace_size(jmix.dims(256, 2, 8192, 256)) == 0
    assert jmix.jm_mixer_step_workspace_size(jmix.dims(256, 1, 8192, 256)) > 0


@pytest.mark.parametrize("bad,code,msg", [
    (dict(d_state=8), jmix.JM_ERR_UNSUPPORTED, "d_state"),
    (dict(d_conv=3), jmix.JM_ERR_UNSUPPORTED, "d_conv"),
    (dict(dt_rank=264), jmix.JM_ERR_UNSUPPORTED, "dt_rank"),
    (dict(d_inner=100), jmix.JM_ERR_INVALID_ARG, "multiples of 8"),
    (dict(dt_rank=12), jmix.JM_ERR_INVALID_ARG, "multiples of 8"),
    (dict(batch=-1), jmix.JM_ERR_INVALID_ARG, "positive"),
    (dict(eps=-1.0), jmix.JM_ERR_INVALID_ARG, "eps"),
    (dict(io=7), jmix.JM_ERR_INVALID_ARG, "io dtype"),
])
def test_rejects_bad_dims(lib, bad, code, msg):
    kw = dict(batch=2, seqlen=16, d_inner=256, dt_rank=16)
    kw.update(bad)
    d = jmix.dims(**kw)
    assert fwd(d) == code
    assert msg in jmix.jm_last_error()


def test_rejects_bad_pointers(lib):
    d = jmix.dims(2, 16, 256, 16)
    assert fwd(d, x=None) == jmix.JM_ERR_INVALID_ARG and "x is NULL" in jmix.jm_last_error()
    assert fwd(d, x=FAKE + 2) == jmix.JM_ERR_INVALID_ARG and "aligned" in jmix.jm_last_error()
    assert fwd(d, y=FAKE) == jmix.JM_ERR_INVALID_ARG and "overlaps" in jmix.jm_last_error()
    assert fwd(d, final_state=None) == jmix.JM_ERR_INVALID_ARG
    assert fwd(d, init_ssm_state=FAKE + 4) == jmix.JM_ERR_INVALID_ARG
    assert fwd(d, ws_bytes=100) == jmix.JM_ERR_WORKSPACE and "too small" in jmix.jm_last_error()
    assert fwd(d, workspace=FAKE + 16) == jmix.JM_ERR_WORKSPACE
    assert fwd(d, workspace=None) == jmix.JM_ERR_WORKSPACE


def test_step_rejects_seqlen_and_missing_state(lib):
    W = {k: FAKE for k in jmix.WEIGHT_NAMES}
    d = jmix.dims(4, 2, 256, 16)
    st = jmix.jm_mixer_step(d, FAKE, FAKE, FAKE, FAKE, W, FAKE + (1 << 36), FAKE, 1 << 30,
                            stream=0, check=False)
    assert st == jmix.JM_ERR_INVALID_ARG and "seqlen" in jmix.jm_last_error()
    d = jmix.dims(4, 1, 256, 16)
    st = jmix.jm_mixer_step(d, FAKE, FAKE, None, FAKE, W, FAKE + (1 << 36), FAKE, 1 << 30,
                            stream=0, check=False)
    assert st == jmix.JM_ERR_INVALID_ARG


def test_binding_raises_on_error(lib):
    with pytest.raises(jmix.JmixError) as e:
        W = {k: FAKE for k in jmix.WEIGHT_NAMES}
        jmix.jm_mixer_fwd(jmix.dims(1, 4, 256, 16, d_conv=2), FAKE, FAKE, W, FAKE, FAKE, FAKE,
                          1 << 30, stream=0)
    assert e.value.status == jmix.JM_ERR_UNSUPPORTED


@pytest.mark.parametrize("B,L,d,io,want", [
    (8, 4096, 8192, jmix.JM_BF16, (4, False)),     # 512 pairs on 296 CTA slots: 4 chained parts
    (1, 4096, 8192, jmix.JM_BF16, (8, True)),      # 64 pairs: state pass + output pass
    (1, 262144, 8192, jmix.JM_BF16, (8, True)),
    (3, 4096, 8192, jmix.JM_BF16, (1, False)),     # 192 pairs: one wave already
    (160, 2100, 256, jmix.JM_BF16, (4, False)),
    (1, 2200, 256, jmix.JM_BF16, (4, True)),
    (2, 1100, 384, jmix.JM_BF16, (2, True)),
    (1, 4200, 200, jmix.JM_BF16, (8, True)),
    (2, 300, 384, jmix.JM_BF16, (1, False)),       # too short to cut
    (8, 4096, 8192, jmix.JM_F32, (1, False)),      # float32 path: one part
])
def test_scan_schedule(lib, B, L, d, io, want):
    assert jmix.jm_mixer_fwd_schedule(jmix.dims(B, L, d, 256 if d == 8192 else 16, io=io)) == want


def test_scan_schedule_rules(lib):
    """Parts hold at least 16 chunks of 32 tokens; chained parts are only used with
    more pairs than CTA slots (two per SM on 148 SMs), where they shorten the last
    wave; the two-pass schedule only with fewer pairs than half the slots."""
    slots = 296
    for B in (1, 2, 5, 8, 16, 64, 160, 300):
        for L in (1, 31, 512, 1023, 1024, 2048, 4096, 9000):
            for d in (128, 200, 1024, 8192):
                n, two = jmix.jm_mixer_fwd_schedule(jmix.dims(B, L, d, 16))
                assert n in (1, 2, 4, 8)
                chunks = -(-L // 32)
                if n > 1:
                    assert chunks >= 16 * n
                pairs = B * -(-d // 128)
                if two:
                    assert pairs < slots // 2
                elif n > 1:
                    assert pairs > slots
                    waves = lambda P: -(-pairs * P // slots) / P
                    assert waves(n) < waves(1)
    with pytest.raises(jmix.JmixError):
        jmix.jm_mixer_fwd_schedule(jmix.dims(1, 10, 100, 16))   # d % 8 != 0


@pytest.mark.parametrize("B,L,d,want", [
    (1, 4096, 8192, 13),   # 64 CTAs per part: 13 parts fill two waves of 444 slots to 94%
    (8, 4096, 8192, 6),    # 512 CTAs per part: 6 parts, 3072 CTAs in 7 waves (99%)
    (4, 4096, 8192, 5),
    (1, 1000, 1024, 16),
    (2, 301, 384, 16),     # 76 chunks: 16 ragged parts of 4-5 chunks
    (2, 37, 200, 1),       # tiny: the folds cost more than the parallelism saves
    (3, 4, 128, 1),        # one chunk
    (1, 0, 8192, 1),       # empty sequences
])
def test_scan_bwd_schedule(lib, B, L, d, want):
    assert jmix.jm_scan_bwd_schedule(jmix.dims(B, L, d, 8)) == want


def test_scan_bwd_schedule_rules(lib):
    """At most 16 parts of at least 2 four-token chunks; one part when the
    (tile, sequence) CTAs already fill 90% of their waves (3 CTAs per SM on 148
    SMs); with parts, the waves are at least as full as with one part."""
    slots = 3 * 148
    fill = lambda ctas: ctas / (-(-ctas // slots) * slots)
    for B in (1, 2, 3, 8, 32, 300):
        for L in (1, 4, 8, 9, 100, 1024, 4096):
            for d in (64, 200, 1024, 8192):
                n = jmix.jm_scan_bwd_schedule(jmix.dims(B, L, d, 8))
                assert 1 <= n <= 16
                chunks = -(-L // 4)
                tiles = -(-d // 128)
                if n > 1:
                    assert chunks >= 2 * n
                    assert fill(tiles * B) < 0.9
                    assert fill(tiles * B * n) >= fill(tiles * B)
    with pytest.raises(jmix.JmixError):
        jmix.jm_scan_bwd_schedule(jmix.dims(1, 10, 128, 8, d_state=8))


def test_scan_bwd_host_checks(lib):
    """jm_scan_bwd validates on the host and returns before any launch."""
    F = 1 << 40          # a fake device address: no test here reaches a launch
    W = 1 << 41          # fake workspace (256-byte aligned)
    d = jmix.dims(2, 64, 256, 8)
    n = jmix.jm_scan_bwd_workspace_size(d)
    assert n > 0 and n % 256 == 0 and n == jmix.jm_scan_bwd_workspace_size(d)

    def call(dm, ws=W, nbytes=n, **over):
        args = dict(delta=F, u=F, Bm=F, Cm=F, A_log=F, D=F, h0=None, gy=F, g_delta=F, g_u=F,
                    g_B=F, g_C=F, g_A_log=F, g_D=F, g_h0=None)
        args.update(over)
        return jmix.jm_scan_bwd(dm, **args, workspace=ws, ws_bytes=nbytes, stream=0, check=False)

    assert call(jmix.dims(2, 64, 256, 8, d_state=8)) == jmix.JM_ERR_UNSUPPORTED
    assert call(jmix.dims(2, 64, 256, 8, zoh=True)) == jmix.JM_ERR_UNSUPPORTED
    assert call(jmix.dims(70000, 4, 128, 8)) == jmix.JM_ERR_INVALID_ARG      # grid y limit
    assert call(jmix.dims(2, 64, 0, 8)) == jmix.JM_ERR_INVALID_ARG
    for k in ("A_log", "D", "g_A_log", "g_D", "delta", "u", "Bm", "Cm", "gy", "g_delta", "g_u",
              "g_B", "g_C"):
        assert call(d, **{k: None}) == jmix.JM_ERR_INVALID_ARG, k
    assert call(d, ws=None) == jmix.JM_ERR_WORKSPACE
    assert call(d, ws=W + 128) == jmix.JM_ERR_WORKSPACE                      # misaligned
    assert call(d, nbytes=n - 256) == jmix.JM_ERR_WORKSPACE                  # too small
    assert jmix.jm_scan_bwd_workspace_size(jmix.dims(2, 64, 256, 8, d_state=8)) == 0
    # more time parts need more per-part rows: the size follows the schedule
    one = jmix.dims(64, 4096, 8192, 8)     # fills the GPU: one part
    assert jmix.jm_scan_bwd_schedule(one) == 1
    parts = jmix.dims(1, 4096, 8192, 8)
    assert jmix.jm_scan_bwd_schedule(parts) > 1
    assert jmix.jm_scan_bwd_workspace_size(parts) > 0


def test_varlen_host_checks(lib):
    FAKE = 1 << 40
    W = {k: FAKE for k in jmix.WEIGHT_NAMES}
    d = jmix.dims(3, 100, 256, 16)
    n = jmix.jm_mixer_fwd_varlen_workspace_size(d)
    assert n > 0
    assert jmix.jm_mixer_fwd_varlen_workspace_size(jmix.dims(3, 100, 256, 16, io=jmix.JM_F32)) == 0
    st = jmix.jm_mixer_fwd_varlen(d, None, FAKE, FAKE, W, FAKE + (1 << 30), FAKE, FAKE, n,
                                  stream=0, check=False)
    assert st == jmix.JM_ERR_INVALID_ARG and "cu_seqlens" in jmix.jm_last_error()
    st = jmix.jm_mixer_fwd_varlen(d, FAKE + 2, FAKE, FAKE, W, FAKE + (1 << 30), FAKE, FAKE, n,
                                  stream=0, check=False)
    assert st == jmix.JM_ERR_INVALID_ARG and "aligned" in jmix.jm_last_error()
    f32 = jmix.dims(3, 100, 256, 16, io=jmix.JM_F32)
    st = jmix.jm_mixer_fwd_varlen(f32, FAKE, FAKE, FAKE, W, FAKE + (1 << 30), FAKE, FAKE, n,
                                  stream=0, check=False)
    assert st == jmix.JM_ERR_UNSUPPORTED
    st = jmix.jm_mixer_fwd_varlen(d, FAKE, FAKE, FAKE, W, FAKE + (1 << 30), FAKE, FAKE, 256,
                                  stream=0, check=False)
    assert st == jmix.JM_ERR_WORKSPACE


def test_discretization_field(lib):
    FAKE = 1 << 40
    W = {k: FAKE for k in jmix.WEIGHT_NAMES}
    d = jmix.dims(2, 10, 256, 16)
    d.discretization = 2
    st = jmix.jm_mixer_fwd(d, FAKE, FAKE + (1 << 30), W, FAKE + (2 << 30), FAKE, FAKE, 1 << 30,
                           stream=0, check=False)
    assert st == jmix.JM_ERR_INVALID_ARG and "discretization" in jmix.jm_last_error()
    d = jmix.dims(2, 10, 256, 16, zoh=True)
    d.reserved = 1
    assert jmix.jm_mixer_fwd_workspace_size(d) == 0
    d.reserved = 0
    assert jmix.jm_mixer_fwd_workspace_size(d) == jmix.jm_mixer_fwd_workspace_size(
        jmix.dims(2, 10, 256, 16))


def test_selftest_timeout_host_checks(lib):
    assert jmix.jm_selftest_timeout(None, 0, stream=0, check=False) == jmix.JM_ERR_WORKSPACE
    assert jmix.jm_selftest_timeout(1 << 40, 128, stream=0, check=False) == jmix.JM_ERR_WORKSPACE


def test_layer_host_checks(lib):
    FAKE = 1 << 40
    W = {k: FAKE for k in jmix.WEIGHT_NAMES}
    d = jmix.dims(2, 10, 256, 16)
    n = jmix.jm_layer_fwd_workspace_size(d, 128)
    assert n > jmix.jm_mixer_fwd_workspace_size(d)
    assert jmix.jm_layer_fwd_workspace_size(d, 100) == 0          # d_model % 8
    assert jmix.jm_layer_fwd_workspace_size(jmix.dims(2, 10, 256, 16, io=jmix.JM_F32), 128) == 0
    st = jmix.jm_layer_fwd(d, 100, FAKE, FAKE, W, FAKE, FAKE, FAKE, FAKE, n, stream=0,
                           check=False)
    assert st == jmix.JM_ERR_INVALID_ARG and "d_model" in jmix.jm_last_error()
    st = jmix.jm_layer_fwd(d, 128, FAKE, FAKE, W, FAKE, FAKE, FAKE, FAKE, n - 256, stream=0,
                           check=False)
    assert st == jmix.JM_ERR_WORKSPACE
    st = jmix.jm_layer_fwd(d, 128, None, FAKE, W, FAKE, FAKE, FAKE, FAKE, n, stream=0,
                           check=False)
    assert st == jmix.JM_ERR_INVALID_ARG and "hidden" in jmix.jm_last_error()


def test_prepare_weights_host_checks(lib):
    d = jmix.dims(2, 1, 8192, 256)
    n = jmix.jm_prepared_weights_size(d)
    assert n == 288 * 8192 * 2 + 8192 * 256 * 2           # both multiples of 256 here
    assert jmix.jm_prepared_weights_size(jmix.dims(2, 1, 8192, 256, jmix.JM_F32)) == 0
    ok = dict(xproj_w=FAKE, dtproj_w=FAKE, prepared=FAKE, nbytes=n)

    def call(dm=d, **over):
        a = dict(ok, **over)
        return jmix.jm_prepare_weights(dm, a["xproj_w"], a["dtproj_w"], a["prepared"],
                                       a["nbytes"], stream=0, check=False)
    assert call(xproj_w=None) == jmix.JM_ERR_INVALID_ARG
    assert call(prepared=FAKE + 16) == jmix.JM_ERR_INVALID_ARG     # not 256-byte aligned
    assert call(nbytes=n - 1) == jmix.JM_ERR_WORKSPACE
    assert call(dm=jmix.dims(2, 1, 8192, 256, jmix.JM_F32)) == jmix.JM_ERR_UNSUPPORTED


def test_indexed_step_host_checks(lib):
    d = jmix.dims(4, 1, 256, 16)
    n = jmix.jm_mixer_step_workspace_size(d)
    W = {k: FAKE for k in jmix.WEIGHT_NAMES}
    ok = dict(idx=FAKE, slots=16, x=FAKE, z=FAKE + (1 << 36), cp=FAKE, sp=FAKE, prep=None,
              y=FAKE + (2 << 36), ws=FAKE, n=n)

    def call(dm=d, **over):
        a = dict(ok, **over)
        return jmix.jm_mixer_step_indexed(dm, a["idx"], a["slots"], a["x"], a["z"], a["cp"],
                                          a["sp"], W, a["prep"], a["y"], a["ws"], a["n"], stream=0,
                                          check=False)
    assert call(idx=None) == jmix.JM_ERR_INVALID_ARG
    assert call(idx=FAKE + 2) == jmix.JM_ERR_INVALID_ARG              # not 4-byte aligned
    assert call(slots=3) == jmix.JM_ERR_INVALID_ARG                   # fewer slots than rows
    assert "n_slots" in jmix.jm_last_error()
    assert call(slots=1 << 31) == jmix.JM_ERR_INVALID_ARG
    assert call(cp=None) == jmix.JM_ERR_INVALID_ARG
    assert call(prep=FAKE + 16) == jmix.JM_ERR_INVALID_ARG           # not 256-byte aligned
    assert call(n=n - 1) == jmix.JM_ERR_WORKSPACE
    assert call(dm=jmix.dims(4, 2, 256, 16)) == jmix.JM_ERR_INVALID_ARG   # seqlen must be 1
    assert call(dm=jmix.dims(4, 1, 256, 16, jmix.JM_F32)) == jmix.JM_ERR_UNSUPPORTED

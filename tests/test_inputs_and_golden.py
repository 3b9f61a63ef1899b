"""CPU checks of the input generator, the workload recipes and the stored fixtures."""
import json
import math
import os

import numpy as np

import oracle
from mamba_selective_scan_jamba_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_generator_matches_numpy_restatement():
    s = synth.stream_seed(3, 1)
    np.testing.assert_array_equal(synth.uniform(s, 4097), synth.np_uniform(s, 4097))
    np.testing.assert_array_equal(synth.uniform(s, 100, start=1000),
                                  synth.np_uniform(s, 1100)[1000:])
    np.testing.assert_allclose(synth.normal(s, 4097), synth.np_normal(s, 4097), rtol=0,
                               atol=1e-14)
    np.testing.assert_array_equal(synth.normal(s, 50, start=100), synth.normal(s, 150)[100:])


def test_generator_statistics():
    n = synth.normal(synth.stream_seed(1, 2), 1 << 20)
    assert abs(n.mean()) < 5e-3 and abs(n.std() - 1) < 5e-3
    u = synth.uniform(synth.stream_seed(1, 3), 1 << 20)
    assert 0 <= u.min() and u.max() < 1 and abs(u.mean() - 0.5) < 2e-3


def test_bf16_encoding():
    v = np.array([1.0, -2.5, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 3.14159, 0.0], dtype=np.float32)
    b = synth.f32_to_bf16_bits(v)
    back = synth.bf16_bits_to_f32(b)
    assert back[0] == 1.0 and back[1] == -2.5 and back[2] == 1.0 and back[3] == 1 + 2 ** -6
    for i in range(len(v)):
        assert back[i] == np.float32(oracle.round_bf16(float(v[i])))


def test_workload_recipes_match_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "jamba_v01_mixer_dims.json")))
    assert g["d_inner"] == 2 * g["d_model"]
    assert g["dt_rank"] == math.ceil(g["d_model"] / 16)
    assert g["x_proj_out"] == g["dt_rank"] + 2 * g["d_state"]
    for name in ("jamba_b1_l4096", "jamba_b8_l4096", "jamba_b1_l262144", "jamba_decode_b256"):
        w = synth.WORKLOADS[name]
        assert (w.d_inner, w.d_state, w.d_conv, w.dt_rank, w.proj) == (
            g["d_inner"], g["d_state"], g["d_conv"], g["dt_rank"], g["x_proj_out"])
        assert w.io == "bf16"
    assert synth.WORKLOADS["jamba_b1_l262144"].seqlen == 256 * 1024
    assert synth.WORKLOADS["jamba_decode_b256"].steps == 64


def test_weight_recipe_statistics():
    w = synth.WORKLOADS["tiny_fp32"].with_(d_inner=512, dt_rank=64)
    W = synth.make_weights(w)
    assert abs(W["xproj_w"].std() - 1 / math.sqrt(512)) < 0.05 / math.sqrt(512)
    assert abs(W["dtproj_w"].std() - 1 / math.sqrt(64)) < 0.05 / math.sqrt(64)
    dt = np.log1p(np.exp(W["dt_bias"].astype(np.float64)))
    assert dt.min() >= 1e-3 * 0.999 and dt.max() <= 1e-1 * 1.001
    np.testing.assert_allclose(-np.exp(W["A_log"][0]), -np.arange(1, 17), rtol=1e-6)
    assert (W["conv_b"] == 0).all() and (W["D"] == 1).all()


def test_oracle_regression_golden():
    g = json.load(open(os.path.join(GOLDEN, "tiny_fp32_oracle.json")))
    for key, extra in (("plain", False), ("extra", True)):
        w = synth.WORKLOADS["tiny_fp32"].with_(extra=extra)
        W = synth.make_weights(w)
        A = synth.make_activations(w)
        y, fs, _ = oracle.mixer_fwd(oracle.dims_of(w), A["x"], A["z"], W,
                                    A.get("init_conv_state"), A.get("init_ssm_state"))
        for idx, v in g[key]["y"]:
            assert abs(y[tuple(idx)] - v) <= 1e-12 * max(1, abs(v))
        for idx, v in g[key]["final_state"]:
            assert abs(fs[tuple(idx)] - v) <= 1e-12 * max(1, abs(v))
        assert abs(np.abs(y).sum() - g[key]["y_abs_sum"]) <= 1e-9 * g[key]["y_abs_sum"]

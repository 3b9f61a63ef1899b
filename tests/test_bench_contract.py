"""CPU checks of bench.py: the per-token work the rooflines divide by, the
per-kernel accounting of the dominant kernel, the packed-batch length recipe,
and the JSON line of the reference arm (the fp64 oracle timed on the host,
run here on a small workload so that it finishes in seconds)."""
import json
import os
import subprocess
import sys

import pytest

import bench
from mamba_selective_scan_jamba_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_work_per_token_at_jamba_shapes():
    w = synth.WORKLOADS["jamba_b8_l4096"]
    t = bench.work_per_token(w)
    d, R, N = 8192, 256, 16
    assert t["bytes"] == 3 * d * 2 == 49152                       # x, z in; y out (bf16)
    assert t["tc_flop"] == 2 * d * (R + 2 * N) + 2 * R * d == 8912896
    assert t["exp"] == d * N == 131072
    f32 = bench.work_per_token(synth.WORKLOADS["tiny_fp32"])
    assert f32["bytes"] == 3 * 128 * 4


def test_kernel_units():
    w = synth.WORKLOADS["jamba_b8_l4096"]
    n = 1000
    assert bench.kernel_units("k_scan_fused", w, n) == ("alu", n * 8192 * 16, "Gexp/s")
    assert bench.kernel_units("k_xproj", w, n) == ("tensor", n * 2 * 8192 * 288, "TFLOP/s")
    assert bench.kernel_units("k_conv_silu16", w, n) == ("hbm", n * 8192 * 2 * 2, "GB/s")
    assert bench.kernel_units("k_norms16", w, n)[0] == "hbm"


def test_varlen_lengths_recipe():
    lens = bench.varlen_lengths()
    assert len(lens) == bench.VARLEN_SEQS and sum(lens) == bench.VARLEN_TOKENS
    assert min(lens) >= 1 and max(lens) <= 8192 * 2
    assert lens == bench.varlen_lengths()          # seeded: the same every time


def test_oracle_sample_shapes():
    w = synth.WORKLOADS["jamba_b8_l4096"]
    assert bench.oracle_sample(w, 100) == (1, 100)           # a prefix of sequence 0
    assert bench.oracle_sample(w, 3 * 4096) == (3, 4096)     # whole sequences
    assert bench.oracle_sample(w, 1e9) == (8, 4096)          # at most the workload


def test_bench_config_names_the_workload():
    w = synth.WORKLOADS["jamba_b8_l4096"]
    c = bench.bench_config(w, 2)
    assert c["workload"] == "jamba_b8_l4096" and c["batch_per_gpu"] == 8 and c["seqlen"] == 4096
    assert c["d_inner"] == 8192 and c["d_state"] == 16 and c["dt_rank"] == 256
    assert "x2" in c["parallelism"] and "L2" in c["l2"]


@pytest.mark.timeout(600)
def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_fp32",
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 0
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["config"]["workload"] == "tiny_fp32"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0

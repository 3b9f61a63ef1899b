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


def test_roofline_block_leads_with_the_stated_fraction(tmp_path, monkeypatch):
    """frac is the step against max(projection FLOPs / bf16 peak, bytes / HBM); the
    dominant kernel's HBM and ALU fractions follow, labelled, with the ALU peak
    from the committed pipe-rate record when there is one."""
    w = synth.WORKLOADS["jamba_b8_l4096"]
    P = dict(hbm=6531.3, bf16=1632.8, bf16_sust=1361.8, sm_max=1965.0, src="measured")
    names = ["k_conv_silu16", "k_xproj", "k_norms16", "k_scan_fused"]
    ms = [0.27, 0.18, 0.02, 2.12]
    tokens = 8 * 4096
    tok_s = tokens / (sum(ms) / 1e3)
    r = bench.roofline_block(P, w, names, ms, tok_s, tokens)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == P["hbm"]
    assert abs(r["achieved"] - tok_s * 49152 / 1e9) < 1e-6
    assert abs(r["frac"] - tok_s / r["roofline_tokens_per_s"]) < 1e-12
    dom = r["dominant_kernel"]
    assert dom["kernel"] == "k_scan_fused"
    assert abs(dom["hbm"]["frac"] - dom["hbm"]["achieved"] / P["hbm"]) < 1e-12
    exps = tokens * 8192 * 16
    assert abs(dom["alu"]["achieved"] - exps / 2.12e-3 / 1e9) < 1e-6
    # without a pipe-rate record the nominal rate is used, and said so
    monkeypatch.setattr(bench, "PIPES_JSON", str(tmp_path / "none.json"))
    r2 = bench.roofline_block(P, w, names, ms, tok_s, tokens)
    assert r2["dominant_kernel"]["alu"]["peak_source"].startswith("nominal")
    assert abs(r2["dominant_kernel"]["alu"]["peak"] - 16 * 148 * 1.965) < 1e-9


def test_traffic_record_is_keyed_to_the_kernel_source(tmp_path):
    p = tmp_path / "traffic.json"
    sha = bench.kernel_source_sha()
    p.write_text(json.dumps({"k_scan_fused": {"bytes_per_token": 51000.5, "source_sha256": sha,
                                              "workload": "w", "capture": "c"},
                             "k_xproj": {"bytes_per_token": 10, "source_sha256": "0" * 64}}))
    got, rec = bench.measured_traffic("k_scan_fused", 1000, str(p))
    assert got == 51000500 and rec["workload"] == "w"
    assert bench.measured_traffic("k_xproj", 1000, str(p)) == (None, None)   # stale source
    assert bench.measured_traffic("k_conv_silu16", 1000, str(p)) == (None, None)

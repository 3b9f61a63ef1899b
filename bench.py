"""Benchmark of the Jamba Mamba-1 mixer core (libjmix) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl jmix|reference]
                    [--workload jamba_b8_l4096] [--no-cpu-baseline] [--no-e2e]

One step = one jm_mixer_fwd over the workload's whole batch (conv + SiLU,
x_proj, RMSNorms, dt_proj + softplus, selective scan, D skip, SiLU(z) gate,
final states), inputs already in HBM.  Under torchrun each rank runs its own
batch (independent sequences, no collective on the data path: weak scaling);
time is the max over ranks of the CUDA-event time on the launching stream.
Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference that exists for
this path) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mamba_selective_scan_jamba_b200.clocks import ClockSampler, gpu_id_of  # noqa: E402

METRIC = "Mamba-mixer tokens/sec at Jamba shapes (d_inner 8192, N 16) and % of roofline"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="jmix", choices=["jmix", "reference"])
    ap.add_argument("--workload", default="jamba_b8_l4096")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--zoh", action="store_true",
                    help="discretise B by zero-order hold instead of delta B")
    ap.add_argument("--bwd", action="store_true",
                    help="also time the scan-core backward (B=1 and B=8, L=4096, d_inner 8192)")
    ap.add_argument("--layer", action="store_true",
                    help="also time the full layer (in_proj -> mixer -> out_proj, d_model 4096)")
    ap.add_argument("--varlen", action="store_true",
                    help="also time jm_mixer_fwd_varlen on a packed batch of mixed lengths")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's sequence length (profiling captures)")
    ap.add_argument("--record-traffic", default="",
                    help="ncu CSV (dram__bytes_read.sum, dram__bytes_write.sum per launch) of "
                         "one jm_mixer_fwd of this workload: write profiles/traffic.json and exit")
    ap.add_argument("--capture", default="", help="the ncu command that made --record-traffic")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return dict(hbm=m["hbm_gbs"], bf16=m["bf16_tflops"],
                    bf16_sust=m["bf16_tflops_sustained"], sm_max=m.get("sm_max_mhz", 1965.0),
                    src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, sm_max=1965.0, src="fallback")


# ----------------------------------------------------------------- per-unit work
def work_per_token(w):
    """Algorithmic work per token (a token = one position across all d_inner channels)."""
    d, R, N = w.d_inner, w.dt_rank, w.d_state
    es = 2 if w.io == "bf16" else 4
    return dict(bytes=3 * d * es,                       # x, z in; y out
                tc_flop=2 * d * (R + 2 * N) + 2 * R * d,  # x_proj + dt_proj
                exp=d * N)                              # scan decays


def kernel_units(name, w, tokens):
    """(bound, algorithmic amount, unit) of one launch of a kernel over `tokens` tokens."""
    d, R, N = w.d_inner, w.dt_rank, w.d_state
    es = 2 if w.io == "bf16" else 4
    if "scan" in name:
        return "alu", tokens * d * N, "Gexp/s"
    if "x_proj" in name or "xproj" in name:
        return "tensor", tokens * 2 * d * (R + 2 * N), "TFLOP/s"
    if "dt_proj" in name:
        return "tensor", tokens * 2 * R * d, "TFLOP/s"
    if "conv" in name:
        return "hbm", tokens * d * es * 2, "GB/s"     # x in, u out
    return "hbm", tokens * (R + 2 * N) * 4 * 2, "GB/s"


def nvtx_push(msg: str) -> None:
    """NVTX range for profilers (a no-op where torch has no NVTX support)."""
    try:
        import torch
        torch.cuda.nvtx.range_push(msg)
    except Exception:  # noqa: BLE001 - tracing must never stop a measurement
        pass


def nvtx_pop() -> None:
    try:
        import torch
        torch.cuda.nvtx.range_pop()
    except Exception:  # noqa: BLE001
        pass


TRAFFIC_JSON = os.path.join(HERE, "profiles", "traffic.json")
PIPES_JSON = os.path.join(HERE, "profiles", "pipe_rates_b200.json")


def kernel_source_sha() -> str:
    src = os.path.join(HERE, "mamba_selective_scan_jamba_b200", "csrc", "k_fast.cu")
    with open(src, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def measured_traffic(kernel: str, tokens: int, path: str = TRAFFIC_JSON):
    """DRAM bytes of one launch of `kernel` over `tokens` tokens from the committed
    ncu record (profiles/traffic.json: bytes per token of a capture, scaled by the
    tokens of this launch), if the kernel source is unchanged since the capture;
    else (None, None)."""
    try:
        with open(path) as f:
            recs = json.load(f)
    except (OSError, ValueError):
        return None, None
    # a launch name may be the family of the recorded kernel (k_norms16 -> k_norms16_warp)
    rec = recs.get(kernel) or next((v for k, v in sorted(recs.items())
                                    if k.startswith(kernel + "_")), None)
    if not rec or rec.get("source_sha256") != kernel_source_sha():
        return None, None
    return int(round(rec["bytes_per_token"] * tokens)), rec


def record_traffic(csv_path: str, w, capture: str, path: str = TRAFFIC_JSON) -> dict:
    """profiles/traffic.json from an ncu CSV of one forward call: DRAM bytes per
    token of each kernel (read + write, summed over its launches in the CSV and
    divided by their tokens), keyed to the current kernel source."""
    import csv
    tokens = w.batch * w.seqlen
    per = {}
    with open(csv_path) as f:
        rows = [r for r in csv.reader(l for l in f if l.startswith('"'))]
    head = rows[0]
    ki, mi, vi, ii = (head.index("Kernel Name"), head.index("Metric Name"),
                      head.index("Metric Value"), head.index("ID"))
    launches = {}
    for r in rows[1:]:
        if r[mi] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            name = re.sub(r"^(void )?(unnamed>::)?", "", r[ki]).split("(")[0].split("<")[0]
            name = name.replace("jmix::", "").strip()
            per[name] = per.get(name, 0.0) + float(r[vi].replace(",", ""))
            launches.setdefault(name, set()).add(r[ii])
    sha = kernel_source_sha()
    out = {}
    for name, b in per.items():
        out[name] = {"bytes_per_token": b / len(launches[name]) / tokens, "source_sha256": sha,
                     "workload": f"{w.name} (B={w.batch}, L={w.seqlen}, {tokens} tokens)",
                     "capture": capture, "launches": len(launches[name]),
                     "metric": "dram__bytes_read.sum + dram__bytes_write.sum"}
    with open(path, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
        f.write("\n")
    return out


def alu_peak(P):
    """(ex2 per second, where it comes from): the measured MUFU ex2 rate of the
    committed pipe-rate record, else the nominal 16 per clock per SM at the
    maximum clock (said so in the source string)."""
    try:
        with open(PIPES_JSON) as f:
            rec = json.load(f)
        rate = float(rec["rates"]["ex2"]["ops_per_s"])
        mhz = rec.get("clocks", {}).get("sm_mhz")
        return rate, (f"measured: profiles/pipe_rates_b200.json (ex2.approx on all SMs, "
                      f"SM clock {mhz} MHz)")
    except (OSError, ValueError, KeyError, TypeError):
        return 16 * 148 * P["sm_max"] * 1e6, (f"nominal: 16 ex2/clk/SM x 148 SMs x "
                                              f"{P['sm_max']:.0f} MHz (no measured record)")


# ------------------------------------------------------------------ decode
def decode_bench(dev, stream, steps: int = 64, warmup: int = 5, zoh: bool = False,
                 pool_slots: int = 0):
    """64 consecutive decode steps on the decode workload (B=256 sequences at Jamba
    shapes, states updated in place); returns a dict for the JSON line.  With
    pool_slots > 0 the steps are jm_mixer_step_indexed calls whose 256 rows use
    distinct, permuted slots of a pool of that many slots (a fresh set every
    step), with the weights prepared once; else jm_mixer_step calls."""
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix, synth
    w = synth.WORKLOADS["jamba_decode_b256"].with_(zoh=zoh)
    W = synth.make_weights(w)
    S = synth.make_decode_state(w.with_(batch=pool_slots) if pool_slots else w)
    Wd = devio.weights_to_device(W, dev)
    cs = devio.to_device(S["conv_state"], dev)
    ss = devio.to_device(S["ssm_state"], dev)
    toks = [synth.make_decode_token(w, t) for t in range(4)]
    xs = [devio.to_device(t["x_t"], dev) for t in toks]
    zs = [devio.to_device(t["z_t"], dev) for t in toks]
    y = torch.empty_like(xs[0])
    d = devio.dims_of(w)
    n = jmix.jm_mixer_step_workspace_size(d)
    ws = devio.workspace(n, dev)
    if pool_slots:
        rng = np.random.default_rng(3)
        idxs = [torch.from_numpy(rng.permutation(pool_slots)[:w.batch].astype(np.int32)).to(dev)
                for _ in range(4)]
        npw = jmix.jm_prepared_weights_size(d)
        prep = devio.workspace(npw, dev)
        jmix.jm_prepare_weights(d, Wd["xproj_w"], Wd["dtproj_w"], prep, npw, stream=stream)

        def one(i):
            jmix.jm_mixer_step_indexed(d, idxs[i % 4], pool_slots, xs[i % 4], zs[i % 4], cs, ss,
                                       Wd, prep, y, ws, n, stream=stream)
    else:
        def one(i):
            jmix.jm_mixer_step(d, xs[i % 4], zs[i % 4], cs, ss, Wd, y, ws, n, stream=stream)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            one(i)
    stream.synchronize()
    nk = jmix.jm_last_launch_count()
    names = [jmix.jm_last_kernel_name(i) for i in range(nk)]
    # the steps back to back, as a serving loop issues them (an event between
    # two kernels would cut the programmatic launch overlap between them)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for i in range(steps):
            one(i)
        b.record(stream)
    stream.synchronize()
    ms = a.elapsed_time(b) / steps
    # then once more with an event around every kernel, for the breakdown
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(steps)]
    with torch.cuda.stream(stream):
        for row in evs:
            for e in row:
                e.record(stream)
    stream.synchronize()
    with torch.cuda.stream(stream):
        for i in range(steps):
            jmix.jm_set_kernel_events([e.cuda_event for e in evs[i]])
            one(i)
    jmix.jm_set_kernel_events(None)
    stream.synchronize()
    assert jmix.jm_poll_error(ws, stream) == jmix.JM_OK, jmix.jm_last_error()
    per = {names[k]: round(sum(evs[i][k].elapsed_time(evs[i][k + 1]) for i in range(steps))
                           / steps * 1e3, 2) for k in range(nk)}
    # algorithmic bytes per step: ssm state r+w, conv state r+w, x_t, z_t, y_t, and
    # every weight read once
    B, dd, N = w.batch, w.d_inner, w.d_state
    wbytes = sum(int(v.nbytes) for v in W.values())
    nbytes = B * dd * (N * 4 * 2 + 3 * 2 * 2 + 2 * 3) + wbytes
    api = (f"jm_mixer_step_indexed: {B} rows in a {pool_slots}-slot pool, permuted slots, "
           "weights prepared once" if pool_slots else "jm_mixer_step")
    return {"workload": w.name, "api": api, "batch": B, "steps": steps, "us_per_step": ms * 1e3,
            "tokens_per_s": B / (ms / 1e3), "algorithmic_bytes_per_step": nbytes,
            "weight_bytes_per_step": wbytes,
            "achieved_GBps": nbytes / (ms / 1e3) / 1e9, "kernels_us": per,
            "kernels_us_note": "a second pass with an event between kernels (no launch overlap)",
            "launches_per_step": nk}


VARLEN_SEQS, VARLEN_TOKENS = 16, 32768


def varlen_lengths(n: int = VARLEN_SEQS, total: int = VARLEN_TOKENS, seed: int = 11):
    """Seeded prompt lengths for the packed-batch measurement: log-uniform in
    [256, 8192] (SplitMix64 uniforms from synth), scaled to `total` tokens."""
    from mamba_selective_scan_jamba_b200 import synth
    u = synth.np_uniform(synth.stream_seed(seed, 99), n)
    raw = np.exp(np.log(256.0) + u * (np.log(8192.0) - np.log(256.0)))
    lens = np.maximum(1, np.floor(raw * total / raw.sum())).astype(np.int64)
    lens[-1] += total - int(lens.sum())
    return [int(v) for v in lens]


def varlen_bench(dev, stream, steps: int = 20, warmup: int = 3):
    """jm_mixer_fwd_varlen on a packed batch of VARLEN_SEQS prompts of mixed lengths
    (VARLEN_TOKENS tokens in all) at Jamba shapes; returns a dict for the JSON line."""
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix, synth
    lens = varlen_lengths()
    T = sum(lens)
    base = synth.WORKLOADS["jamba_b8_l4096"]
    w = base.with_(name="jamba_varlen", batch=1, seqlen=T)
    W = synth.make_weights(base)
    A = synth.make_activations(w)
    Wd = devio.weights_to_device(W, dev)
    x = devio.to_device(A["x"][0], dev)
    z = devio.to_device(A["z"][0], dev)
    y = torch.empty_like(x)
    B = len(lens)
    fs = torch.empty((B, w.d_inner, w.d_state), dtype=torch.float32, device=dev)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    d = jmix.dims(B, T, w.d_inner, w.dt_rank, jmix.JM_BF16, w.eps)
    n = jmix.jm_mixer_fwd_varlen_workspace_size(d)
    ws = devio.workspace(n, dev)

    def step():
        jmix.jm_mixer_fwd_varlen(d, cu, x, z, Wd, y, fs, ws, n, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    stream.synchronize()
    nk = jmix.jm_last_launch_count()
    names = [jmix.jm_last_kernel_name(i) for i in range(nk)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(steps)]
    with torch.cuda.stream(stream):
        for row in evs:
            for e in row:
                e.record(stream)
    stream.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for i in range(steps):
            jmix.jm_set_kernel_events([e.cuda_event for e in evs[i]])
            step()
        b.record(stream)
    jmix.jm_set_kernel_events(None)
    stream.synchronize()
    assert jmix.jm_poll_error(ws, stream) == jmix.JM_OK, jmix.jm_last_error()
    ms = a.elapsed_time(b) / steps
    per = {names[k]: round(sum(evs[i][k].elapsed_time(evs[i][k + 1]) for i in range(steps))
                           / steps, 4) for k in range(nk)}
    return {"workload": "packed prefill at Jamba shapes", "sequences": B, "lengths": lens,
            "tokens": T, "steps": steps, "ms_per_step": ms, "tokens_per_s": T / (ms / 1e3),
            "kernels_ms": per, "launches_per_step": nk}


def layer_bench(dev, stream, w, d_model: int = 4096, steps: int = 10, warmup: int = 3,
                mixer_ms: float = 0.0):
    """jm_layer_fwd (in_proj -> mixer core -> out_proj, both projections on libjmix's
    tcgen05 GEMM) on the workload at Jamba's d_model; returns a dict for the JSON
    line.  mixer_ms (the mixer core alone, timed by the caller on the same
    workload) splits the layer's time into mixer and projections."""
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix, synth
    W = synth.make_weights(w)
    LW = synth.make_layer(w, d_model)
    Wd = devio.weights_to_device(W, dev)
    hid = devio.to_device(LW["hidden"], dev)
    wi, wo = devio.to_device(LW["in_proj_w"], dev), devio.to_device(LW["out_proj_w"], dev)
    out = torch.empty_like(hid)
    fs = torch.empty((w.batch, w.d_inner, w.d_state), dtype=torch.float32, device=dev)
    d = devio.dims_of(w)
    n = jmix.jm_layer_fwd_workspace_size(d, d_model)
    ws = devio.workspace(n, dev)

    def step():
        jmix.jm_layer_fwd(d, d_model, hid, wi, Wd, wo, out, fs, ws, n, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    stream.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
    stream.synchronize()
    assert jmix.jm_poll_error(ws, stream) == jmix.JM_OK, jmix.jm_last_error()
    ms = a.elapsed_time(b) / steps
    T = w.batch * w.seqlen
    gemm_flop = 2.0 * T * d_model * 3 * w.d_inner        # in_proj (2 d_inner) + out_proj
    out = {"workload": f"{w.name} + in_proj/out_proj (d_model {d_model})", "tokens": T,
           "steps": steps, "ms_per_step": ms, "tokens_per_s": T / (ms / 1e3),
           "projection_tflop_per_step": gemm_flop / 1e12,
           "projections": "k_gemm_bf16: tcgen05 bf16 GEMM, fp32 accumulation in TMEM; in_proj "
                          "writes x and z in the mixer's layout"}
    if mixer_ms > 0:
        proj_ms = ms - mixer_ms
        out.update({"mixer_ms": mixer_ms, "projections_ms": proj_ms,
                    "projection_tflops": gemm_flop / (proj_ms / 1e3) / 1e12})
    return out


def bwd_bench(dev, stream, B: int = 1, L: int = 4096, d: int = 8192, steps: int = 5,
              warmup: int = 2):
    """jm_scan_bwd (backward of the scan core, float32) at Jamba's d_inner; returns a
    dict for the JSON line."""
    import torch
    from mamba_selective_scan_jamba_b200 import devio, jmix
    g = torch.Generator(device=dev).manual_seed(7)
    rnd = lambda *s: torch.randn(*s, device=dev, generator=g)
    delta = torch.exp(torch.empty(B, L, d, device=dev).uniform_(math.log(1e-3), math.log(0.1),
                                                                generator=g))
    u, gy = rnd(B, L, d), rnd(B, L, d)
    Bm, Cm = rnd(B, L, 16), rnd(B, L, 16)
    A_log = torch.log(torch.arange(1, 17, device=dev, dtype=torch.float32)).repeat(d, 1)
    D = torch.ones(d, device=dev)
    outs = [torch.empty(B, L, d, device=dev), torch.empty(B, L, d, device=dev),
            torch.empty(B, L, 16, device=dev), torch.empty(B, L, 16, device=dev),
            torch.empty(d, 16, device=dev), torch.empty(d, device=dev),
            torch.empty(B, d, 16, device=dev)]
    dm = jmix.dims(B, L, d, 8)
    n = jmix.jm_scan_bwd_workspace_size(dm)
    ws = devio.workspace(n, dev)

    def step():
        jmix.jm_scan_bwd(dm, delta, u, Bm, Cm, A_log, D, None, gy, *outs, ws, n, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    stream.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
    stream.synchronize()
    assert jmix.jm_poll_error(ws, stream) == jmix.JM_OK, jmix.jm_last_error()
    ms = a.elapsed_time(b) / steps
    return {"workload": f"scan-core backward, B={B}, L={L}, d_inner={d}, float32",
            "tokens": B * L, "ms_per_step": ms, "tokens_per_s": B * L / (ms / 1e3),
            "data": "synthetic (torch generator, seed 7)"}


def roofline_block(P, w, names, per_kernel_ms, tok_s, tokens):
    """The roofline object of the JSON line.  Top level: the whole step against
    the stated roofline, max(projection FLOPs / bf16 peak, x,z,y bytes / HBM) per
    token; at Jamba shapes the HBM term is the larger, so `achieved` is the
    step's algorithmic bytes per second and `frac` the stated fraction.  The
    dominant kernel follows with its own HBM and ALU (MUFU ex2) fractions."""
    wt = work_per_token(w)
    t_hbm = wt["bytes"] / (P["hbm"] * 1e9)
    t_tc = wt["tc_flop"] / (P["bf16_sust"] * 1e12)
    hbm_bound = t_hbm >= t_tc
    roof_tok_s = 1.0 / max(t_hbm, t_tc)
    kd = max(range(len(names)), key=lambda k: per_kernel_ms[k])
    t_k = per_kernel_ms[kd] / 1e3
    kname = names[kd]
    traffic, trec = measured_traffic(kname, tokens)
    dom = {"kernel": kname, "ms": per_kernel_ms[kd], "share_of_step":
           per_kernel_ms[kd] / max(sum(per_kernel_ms), 1e-12)}
    if "scan" in kname:
        # algorithmic bytes of the scan kernel: x, z in, y out, dt_n (fp16) and B/C in
        kb = tokens * (wt["bytes"] + 2 * w.dt_rank + 4 * 2 * w.d_state)
        dom["hbm"] = {"achieved": kb / t_k / 1e9, "peak": P["hbm"], "unit": "GB/s",
                      "frac": kb / t_k / 1e9 / P["hbm"],
                      "algorithmic_bytes_per_token": kb / tokens}
        rate, src = alu_peak(P)
        exps = tokens * wt["exp"]
        dom["alu"] = {"achieved": exps / t_k / 1e9, "peak": rate / 1e9, "unit": "Gexp/s",
                      "frac": exps / t_k / rate, "peak_source": src,
                      "counted": "16 ex2 per (token, channel): the state decays"}
    else:
        bound, amount, unit = kernel_units(kname, w, tokens)
        peak = P["bf16_sust"] if bound == "tensor" else P["hbm"]
        ach = amount / t_k / (1e12 if bound == "tensor" else 1e9)
        dom[bound] = {"achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak}
    dom["traffic"] = traffic
    dom["traffic_source"] = ("profiles/traffic.json: %s (%s), ncu dram__bytes_read.sum + "
                             "dram__bytes_write.sum per token x this launch's tokens"
                             % (trec.get("workload"), trec.get("capture"))
                             if trec else "none for the current kernel source")
    if hbm_bound:
        ach, peak, unit, bound = tok_s * wt["bytes"] / 1e9, P["hbm"], "GB/s", "hbm"
    else:
        ach, peak, unit, bound = tok_s * wt["tc_flop"] / 1e12, P["bf16_sust"], "TFLOP/s", "tensor"
    step_traffic = None
    recs = [measured_traffic(n, tokens)[0] for n in names]
    if all(r is not None for r in recs):
        step_traffic = sum(recs)
    return {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
            "traffic": step_traffic,
            "scope": "whole step (every kernel of one jm_mixer_fwd), stated roofline",
            "definition": "max(x_proj + dt_proj FLOPs / bf16 sustained peak, x,z in + y out "
                          "bytes / HBM) per token",
            "roofline_tokens_per_s": roof_tok_s,
            "peak_source": f"{P['src']} MEASURED_PEAKS.json",
            "kernels_ms": {names[k]: round(per_kernel_ms[k], 4) for k in range(len(names))},
            "dominant_kernel": dom}


# ------------------------------------------------------------- cpu baseline
def oracle_sample(w, tokens: float):
    """(sequences, tokens per sequence) of a sample of about `tokens` tokens taken
    from the start of the workload: a prefix of sequence 0, or whole sequences."""
    tokens = int(max(16, tokens))
    if tokens <= w.seqlen:
        return 1, tokens
    return max(1, min(w.batch, round(tokens / w.seqlen))), w.seqlen


def oracle_rate(w, target_s: float, threads: int = 0):
    """Time the fp64 oracle on a sample of the workload sized so that the run
    takes about target_s seconds.  Returns (tokens/s, cores, sample description)."""
    import oracle
    from mamba_selective_scan_jamba_b200 import synth
    cores = threads or os.cpu_count() or 1
    W = synth.make_weights(w)
    L0 = min(w.seqlen, 64)
    A = synth.make_activations(w.with_(batch=1, seqlen=L0))
    t = time.perf_counter()
    oracle.mixer_fwd(oracle.dims_of(w, batch=1, seqlen=L0, threads=cores), A["x"], A["z"], W)
    dt0 = time.perf_counter() - t
    # the short probe overstates the per-token cost (fixed costs dominate it), so
    # the sample is resized once more from its own time when it ran short
    tokens = L0 * target_s / max(dt0, 1e-3)
    for _ in range(2):
        nb, L = oracle_sample(w, tokens)
        A = synth.make_activations(w.with_(seqlen=L), 0, nb)
        t = time.perf_counter()
        oracle.mixer_fwd(oracle.dims_of(w, batch=nb, seqlen=L, threads=cores), A["x"], A["z"], W)
        dt = time.perf_counter() - t
        if dt >= 0.5 * target_s or nb * L >= w.batch * w.seqlen:
            break
        tokens = nb * L * target_s / max(dt, 1e-3)
    return nb * L / dt, cores, (f"sequences 0..{nb - 1} of {w.name}, first {L} tokens each "
                                f"(B={nb}, L={L}, d_inner={w.d_inner}, dt_rank={w.dt_rank}), "
                                f"fp64 oracle, {cores} threads, {dt:.1f} s")


def bench_config(w, world: int) -> dict:
    """The `config` object of both arms' JSON lines."""
    in_bytes = w.batch * w.seqlen * w.d_inner * (2 if w.io == "bf16" else 4) * 2
    return {"workload": w.name, "batch_per_gpu": w.batch, "seqlen": w.seqlen,
            "d_inner": w.d_inner, "d_state": w.d_state, "dt_rank": w.dt_rank,
            "discretization": "zoh" if w.zoh else "euler",
            "parallelism": f"replicas x{world} (independent sequences)",
            "l2": f"no flush: x+z = {in_bytes / 1e9:.2f} GB per step > 126 MB L2"}


def reference_arm(args, w, rank, world):
    if rank != 0:
        return
    import oracle
    from mamba_selective_scan_jamba_b200 import synth
    cores = os.cpu_count() or 1
    W = synth.make_weights(w)
    # per-step sample sized so that warm-up + timed steps take about two minutes
    per_step_s = min(2.0, 120.0 / max(1, args.steps + args.warmup))
    rate, _, _ = oracle_rate(w, 1.0, cores)
    L = int(max(8, min(w.seqlen, rate * per_step_s)))
    A = synth.make_activations(w.with_(batch=1, seqlen=L))
    m = oracle.dims_of(w, batch=1, seqlen=L, threads=cores)
    for _ in range(args.warmup):
        oracle.mixer_fwd(m, A["x"], A["z"], W)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.mixer_fwd(m, A["x"], A["z"], W)
    dt = (time.perf_counter() - t) / max(1, args.steps)
    value = L / dt
    sample = (f"per step: sequence 0 of {w.name}, first {L} tokens (B=1, L={L}), fp64 oracle "
              f"on {cores} host threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- main
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from mamba_selective_scan_jamba_b200 import synth
    base = synth.WORKLOADS[args.workload]
    if args.seqlen:
        base = base.with_(seqlen=args.seqlen, name=f"{base.name}_L{args.seqlen}")
    if args.zoh:
        base = base.with_(zoh=True, name=f"{base.name}_zoh")
    if args.impl == "reference":
        reference_arm(args, base, rank, world)
        return
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic, base, args.capture), indent=1))
        return

    import torch
    import torch.distributed as dist
    from mamba_selective_scan_jamba_b200 import devio, jmix, replicas

    torch.cuda.set_device(local)
    if world > 1:
        replicas.init("nccl", 120.0, torch.device("cuda", local))
    P = peaks()
    # weak scaling: rank r owns sequences r*B .. r*B+B-1 of a world*B batch
    w = base
    wall = base.with_(batch=base.batch * world)
    W = synth.make_weights(w)
    A = synth.make_activations(wall, *replicas.shard(w.batch, rank))
    dev = torch.device("cuda", local)
    Wd = devio.weights_to_device(W, dev)
    x = devio.to_device(A["x"], dev)
    z = devio.to_device(A["z"], dev)
    y = torch.empty_like(x)
    fs = torch.empty((w.batch, w.d_inner, w.d_state), dtype=torch.float32, device=dev)
    d = devio.dims_of(w)
    nbytes = jmix.jm_mixer_fwd_workspace_size(d)
    ws = devio.workspace(nbytes, dev)
    stream = torch.cuda.Stream(device=dev)
    in_bytes = x.numel() * x.element_size() * 2

    def step():
        jmix.jm_mixer_fwd(d, x, z, Wd, y, fs, ws, nbytes, stream=stream)

    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    nk = jmix.jm_last_launch_count()
    names = [jmix.jm_last_kernel_name(i) for i in range(nk)]
    assert jmix.jm_poll_error(ws, stream) == jmix.JM_OK, jmix.jm_last_error()

    # per-kernel events for every timed step (recorded on the launching stream)
    K, Wm = args.steps, args.warmup
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(K)]
    with torch.cuda.stream(stream):
        for row in evs:           # materialise the events so their handles exist
            for e in row:
                e.record(stream)
    stream.synchronize()
    handles = [[e.cuda_event for e in row] for row in evs]

    with torch.cuda.stream(stream):
        for _ in range(Wm):
            step()
    stream.synchronize()
    sampler = ClockSampler(gpu_id_of(dev))
    time.sleep(0.6)   # let the sampler start
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    replicas.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    launches = 0
    nvtx_push(f"jmix timed region: {K} x jm_mixer_fwd ({w.name})")
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(K):
            jmix.jm_set_kernel_events(handles[i])
            step()
            launches += jmix.jm_last_launch_count()
        end.record(stream)
    nvtx_pop()
    jmix.jm_set_kernel_events(None)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    replicas.barrier()
    time.sleep(0.3)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    assert jmix.jm_poll_error(ws, stream) == jmix.JM_OK, jmix.jm_last_error()
    ms = start.elapsed_time(end) / K
    per_kernel = [sum(evs[i][k].elapsed_time(evs[i][k + 1]) for i in range(K)) / K
                  for k in range(nk)]
    ms = replicas.max_over_ranks(ms, dev)
    tokens_rank = w.batch * w.seqlen
    value = replicas.job_rate(tokens_rank, world, ms)

    roofline = roofline_block(P, w, names, per_kernel, value / world, tokens_rank)

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": Wm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.io == "bf16" else "f32",
            "data": "synthetic",
            "config": bench_config(w, world),
            "roofline": roofline, "gpu_launches": launches, "clocks": clocks}

    # end to end through the host-buffer entry point
    if not args.no_e2e:
        xh, zh = devio.to_pinned(A["x"]), devio.to_pinned(A["z"])
        yh = torch.empty(x.shape, dtype=x.dtype).pin_memory()
        fsh = torch.empty(fs.shape, dtype=torch.float32).pin_memory()
        Ke = max(1, min(K, 10))

        def e2e_step():
            jmix.jm_mixer_fwd_host(d, xh, zh, yh, fsh, x, z, y, fs, Wd, ws, nbytes,
                                   stream=stream)

        with torch.cuda.stream(stream):
            e2e_step()
        stream.synchronize()
        replicas.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            s2.record(stream)
            for _ in range(Ke):
                e2e_step()
            e2.record(stream)
        stream.synchronize()
        ems = replicas.max_over_ranks(s2.elapsed_time(e2) / Ke, dev)
        line["e2e"] = {"value": replicas.job_rate(tokens_rank, world, ems), "unit": "tokens/s",
                       "h2d_bytes_per_step": in_bytes,
                       "d2h_bytes_per_step": y.numel() * y.element_size() + fs.numel() * 4,
                       "ms_per_step": ems, "steps": Ke,
                       "api": "jm_mixer_fwd_host (pinned host x, z -> y, final_state)"}

    if args.varlen:
        line["varlen"] = varlen_bench(dev, stream)
    if args.layer:
        line["layer"] = layer_bench(dev, stream, w, mixer_ms=ms)
    if args.bwd:
        line["bwd"] = [bwd_bench(dev, stream, B=1), bwd_bench(dev, stream, B=8)]
    if not args.no_decode:
        dec = decode_bench(dev, stream, zoh=args.zoh)
        dec["hbm_frac"] = dec["achieved_GBps"] / P["hbm"]
        line["decode"] = dec
        ind = decode_bench(dev, stream, zoh=args.zoh, pool_slots=1024)
        ind["hbm_frac"] = ind["achieved_GBps"] / P["hbm"]
        line["decode_indexed"] = ind
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, sample = oracle_rate(w, 12.0)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        replicas.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Measured pipe rates of the GPU the selective scan runs on.

    python -m mamba_selective_scan_jamba_b200.pipe_rates [--out profiles/pipe_rates_b200.json]

Times each microbenchmark of ``csrc/pipe_rates.cu`` (MUFU ex2 / tanh / rcp, FFMA,
packed FFMA2, and ex2 interleaved with FFMA2) on every SM at full occupancy with
CUDA events, samples the SM clock with nvidia-smi meanwhile, and writes one JSON
record: operations per second and per clock per SM for each op.  The scan's ALU
roofline divides its 16 ex2 per (token, channel) by the measured ex2 rate.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
DEFAULT_OUT = os.path.join(ROOT, "profiles", "pipe_rates_b200.json")

# op code -> (name, operations per lane per instruction, what is counted)
OPS = {0: ("ex2", 1, "ex2.approx.ftz.f32"), 1: ("tanh", 1, "tanh.approx.f32 (+1 add)"),
       2: ("rcp", 1, "rcp.approx.ftz.f32 (+1 add)"), 3: ("ffma", 1, "fma.rn.f32"),
       4: ("ffma2", 2, "fma.rn.f32x2, 2 FMAs per lane"),
       5: ("ex2_with_2ffma2", 1, "ex2 counted; 2 fma.rn.f32x2 issued beside each")}
# the scan's recurrence alone: 16 ex2 per token and thread (counted per ex2)
RECURRENCE = {6: ("recurrence_bc_smem", 16, "16-state update, B/C rows from shared memory"),
              7: ("recurrence_bc_regs", 16, "16-state update, B/C in registers")}


def source_sha256() -> str:
    with open(os.path.join(HERE, "csrc", "pipe_rates.cu"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def measure(target_ms: float = 60.0, reps: int = 5) -> dict:
    import torch
    from . import build
    from .clocks import ClockSampler, gpu_id_of
    lib = ctypes.CDLL(build.build_pipes())
    lib.jmp_launch.restype = ctypes.c_int
    lib.jmp_launch.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                               ctypes.c_void_p, ctypes.c_void_p]
    chains = lib.jmp_chains()
    dev = torch.device("cuda", torch.cuda.current_device())
    props = torch.cuda.get_device_properties(dev)
    sms = props.multi_processor_count
    threads, blocks = 256, sms * 8           # 64 warps per SM: full occupancy
    sink = torch.zeros(threads, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def run(op, iters, nb, nt):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            rc = lib.jmp_launch(op, nb, nt, iters, ctypes.c_void_p(sink.data_ptr()),
                                ctypes.c_void_p(stream.cuda_stream))
            b.record(stream)
        assert rc == 0, f"launch failed ({rc})"
        stream.synchronize()
        return a.elapsed_time(b)

    sampler = ClockSampler(gpu_id_of(dev))
    time.sleep(0.5)
    t0 = time.time()
    rates = {}
    # every op at full occupancy (64 warps per SM), then ex2 and ex2 beside FFMA2
    # at the scan kernel's occupancy (8 compute warps per SM: 2 per scheduler)
    cases = [(op, name, per_lane, what, blocks, threads) for op, (name, per_lane, what)
             in OPS.items()]
    cases += [(op, OPS[op][0] + "_2warps_per_smsp", OPS[op][1], OPS[op][2], sms * 2, 128)
              for op in (0, 5)]
    # the recurrence at the scan kernel's occupancy (2 compute warps per
    # scheduler) and at 4 warps per scheduler
    for op, (name, per_lane, what) in RECURRENCE.items():
        cases.append((op, name + "_2warps_per_smsp", per_lane / chains, what, sms * 2, 128))
        cases.append((op, name + "_4warps_per_smsp", per_lane / chains, what, sms * 4, 128))
    for op, name, per_lane, what, nb, nt in cases:
        iters = 4096
        run(op, iters, nb, nt)              # first launch of this kernel: module load
        ms = run(op, iters, nb, nt)
        iters = max(4096, int(iters * target_ms / max(ms, 1e-3)))
        times = [run(op, iters, nb, nt) for _ in range(reps)]
        ms = statistics.median(times)
        ops = float(nb) * nt * iters * chains * per_lane
        rates[name] = {"ops_per_s": ops / (ms / 1e3), "what": what, "iters": iters,
                       "ms_median": ms, "blocks": nb, "threads": nt}
    t1 = time.time()
    time.sleep(0.3)
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    mhz = clocks.get("sm_mhz") or 0.0
    for name, r in rates.items():
        r["per_clk_per_sm"] = r["ops_per_s"] / (mhz * 1e6 * sms) if mhz else None
        # a launch that took far less than intended did not do the work it counts
        assert r["ms_median"] > 0.25 * target_ms, (name, r)
    return {"gpu": props.name, "sms": sms, "chains_per_thread": chains, "clocks": clocks, "rates": rates,
            "source": "mamba_selective_scan_jamba_b200/csrc/pipe_rates.cu",
            "source_sha256": source_sha256(),
            "command": "python -m mamba_selective_scan_jamba_b200.pipe_rates --out "
                       "profiles/pipe_rates_b200.json"}


def load(path: str = DEFAULT_OUT):
    """The committed record, or None."""
    try:
        with open(path) as f:
            return json.load(f)
    except (OSError, ValueError):
        return None


def main(argv=None) -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=DEFAULT_OUT)
    args = ap.parse_args(argv)
    rec = measure()
    with open(args.out, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec))


if __name__ == "__main__":
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    main()

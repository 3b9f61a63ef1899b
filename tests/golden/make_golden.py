"""Writes tests/golden/tiny_fp32_oracle.json: sampled outputs of the fp64 oracle
on the tiny fp32 workload (and its extra-terms variant).  Calls only oracle/ and
the seeded input generator; rerun it only when a change to the oracle's
arithmetic is justified by the pages."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from mamba_selective_scan_jamba_b200 import synth  # noqa: E402

IDX_Y = [(0, 0, 0), (0, 3, 17), (0, 31, 64), (0, 63, 127), (0, 40, 5)]
IDX_S = [(0, 0, 0), (0, 17, 15), (0, 127, 7), (0, 64, 3)]


def compute(extra: bool):
    w = synth.WORKLOADS["tiny_fp32"].with_(extra=extra)
    W = synth.make_weights(w)
    A = synth.make_activations(w)
    y, fs, fc = oracle.mixer_fwd(oracle.dims_of(w), A["x"], A["z"], W, A.get("init_conv_state"),
                                 A.get("init_ssm_state"))
    return {"y": [[list(i), float(y[i])] for i in IDX_Y],
            "final_state": [[list(i), float(fs[i])] for i in IDX_S],
            "y_abs_sum": float(np.abs(y).sum()), "state_abs_sum": float(np.abs(fs).sum())}


def main():
    out = {"_note": "fp64 oracle outputs on the tiny fp32 workload; regression guard for the oracle",
           "plain": compute(False), "extra": compute(True)}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32_oracle.json"),
              "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()

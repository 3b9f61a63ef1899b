"""Planted mistakes in the oracle's dt branch, each caught by a pin (CPU only).

delta = softplus(W_dt . (RMSNorm(dt) w_dt) + dt_bias) is the one part of the
oracle that no closed form of the scan reaches (TransformerLens "Jamba" adapter
page, "Key adapter decisions": the RMSNorms on dt, B and C; aifetchly "Jamba
Guide", "Hands-On Implementation": delta = softplus(dt_proj(.))).  Each case
below copies the oracle's source, plants one plausible mistake in the copy,
builds it into a temporary library and runs the dt-branch pins of
test_oracle_pins.py against it: at least one pin must fail.  The oracle in the
tree is never modified.
"""
import os
import subprocess

import pytest

import oracle
from test_oracle_pins import DT_BRANCH_CHECKS

NORM_DT = "    orc_rmsnorm(1, R, R, p.data(), dtn_w, m->eps, dtn + t * R);\n"
WDT_ROW = "      const double* wr = dtproj_w + ch[i] * R;\n"
WDT_USE = "      for (int64_t r = 0; r < R; ++r) acc += wr[r] * dtn[t * R + r];\n"

PLANTED = {
    # dt_proj applied to the raw dt: the norm skipped, its weight kept
    "norm_skipped": [(NORM_DT, "    for (int64_t r = 0; r < R; ++r) dtn[t * R + r] = p[r] * "
                               "dtn_w[r];\n")],
    # the norm's weight w_dt dropped
    "norm_weight_dropped": [(NORM_DT, "    { std::vector<double> one(R, 1.0);\n"
                                      "      orc_rmsnorm(1, R, R, p.data(), one.data(), m->eps, "
                                      "dtn + t * R); }\n")],
    # the mean of squares taken over all R + 2N x_proj outputs instead of the R dt ones
    "norm_over_all_outputs": [(NORM_DT, "    { double ss = 0.0;\n"
                                        "      for (int64_t j = 0; j < P; ++j) ss += p[j] * p[j];\n"
                                        "      const double inv = 1.0 / std::sqrt(ss / (double)P + "
                                        "m->eps);\n"
                                        "      for (int64_t r = 0; r < R; ++r) dtn[t * R + r] = "
                                        "p[r] * inv * dtn_w[r]; }\n")],
    # W_dt read as [R, d_inner] instead of [d_inner, R]
    "dtproj_transposed": [(WDT_ROW, ""),
                          (WDT_USE, "      for (int64_t r = 0; r < R; ++r) acc += "
                                    "dtproj_w[r * m->d_inner + ch[i]] * dtn[t * R + r];\n")],
}


def _build_variant(src_text: str, edits, out_dir: str, name: str) -> str:
    for old, new in edits:
        assert src_text.count(old) == 1, f"planting {name}: target line not found once: {old!r}"
        src_text = src_text.replace(old, new)
    cpp = os.path.join(out_dir, f"orc_{name}.cpp")
    lib = os.path.join(out_dir, f"liborc_{name}.so")
    with open(cpp, "w") as f:
        f.write(src_text)
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-shared", "-fPIC", "-pthread",
                           "-ffp-contract=off", "-fno-fast-math", cpp, "-o", lib])
    return lib


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_planted_dt_mistake_fails_a_pin(name, tmp_path, monkeypatch):
    with open(oracle.SRC) as f:
        src = f.read()
    lib = oracle.load_library(_build_variant(src, PLANTED[name], str(tmp_path), name))
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = []
    for check in DT_BRANCH_CHECKS:
        try:
            check()
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"planted mistake {name} passed every dt-branch pin"


def test_unplanted_copy_passes_every_pin(tmp_path, monkeypatch):
    """The same build route with no edit passes, so the failures above come from
    the planted mistakes, not from the temporary build."""
    with open(oracle.SRC) as f:
        src = f.read()
    lib = oracle.load_library(_build_variant(src, [], str(tmp_path), "as_is"))
    monkeypatch.setattr(oracle, "_lib", lib)
    for check in DT_BRANCH_CHECKS:
        check()

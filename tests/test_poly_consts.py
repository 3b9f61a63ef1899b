"""CPU checks of the scan kernel's FMA-pipe function constants (csrc/poly_consts.cuh):
they must be what gen_poly.py derives, and the float32 evaluation schemes the
kernel uses must meet their error bounds against float64 references."""
import importlib.util
import os
import re

import numpy as np

from mamba_selective_scan_jamba_b200 import build

GEN = os.path.join(build.CSRC, "gen_poly.py")
HDR = os.path.join(build.CSRC, "poly_consts.cuh")


def header_consts():
    src = open(HDR).read()
    return {k: np.float32(float(v)) for k, v in
            re.findall(r"constexpr float (\w+) = ([-+0-9.eE]+)f;", src)}


def test_header_matches_generator():
    spec = importlib.util.spec_from_file_location("gen_poly", GEN)
    g = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(g)
    assert open(HDR).read() == g.render()


def test_exp2_range_reduction_and_polynomial():
    c = header_consts()
    E = [c["E%d" % i] for i in range(7)]
    x = -np.concatenate([np.linspace(0, 1, 100001), np.geomspace(1e-8, 126, 200001)]).astype(
        np.float32)
    kround = np.float32(12582912.0)
    t = (np.maximum(x, np.float32(-126)) + kround).astype(np.float32)
    j = (t - kround).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = np.float32(E[6])
    for k in range(5, -1, -1):
        p = (p * f + E[k]).astype(np.float32)
    scaled = (p.view(np.int32) + (t.view(np.int32) << np.int32(23))).view(np.float32)
    ref = np.exp2(x.astype(np.float64))
    ok = ref > 2.0 ** -125
    rel = np.abs(scaled[ok] - ref[ok]) / ref[ok]
    assert rel.max() < 2.5e-7, rel.max()
    assert abs(np.mean((scaled[ok] - ref[ok]) / ref[ok])) < 2e-8   # no systematic bias


def test_log1p_polynomial():
    c = header_consts()
    Lc = [c["L%d" % i] for i in range(9)]
    w = np.concatenate([np.linspace(0, 1, 100001), np.geomspace(1e-30, 1, 100001)]).astype(
        np.float32)
    q = np.float32(Lc[8])
    for k in range(7, -1, -1):
        q = (q * w + Lc[k]).astype(np.float32)
    val = (w * q).astype(np.float64)
    ref = np.log1p(w.astype(np.float64))
    ok = w > 0
    assert (np.abs(val[ok] - ref[ok]) / ref[ok]).max() < 3e-7


def test_newton_reciprocal():
    c = header_consts_int()
    K = c["RCP_MAGIC"]
    den = np.concatenate([np.linspace(1, 2, 100001), np.geomspace(1, 8.5e37, 200001)]).astype(
        np.float32)
    r = (np.int64(K) - den.view(np.int32).astype(np.int64)).astype(np.int32).view(np.float32)
    for _ in range(3):   # r * fma(-den, r, 2): the fma is exact to one rounding in float64 here
        e = (2.0 - den.astype(np.float64) * r.astype(np.float64)).astype(np.float32)
        r = (r * e).astype(np.float32)
    rel = np.abs(r.astype(np.float64) * den.astype(np.float64) - 1)
    assert rel.max() < 2e-7, rel.max()


def header_consts_int():
    src = open(HDR).read()
    return {k: int(v, 16) for k, v in re.findall(r"constexpr int (\w+) = (0x[0-9a-fA-F]+);", src)}

"""Build steps for the native parts of the package.

* ``libjmix.so``: the CUDA kernels and the C ABI, compiled for sm_100a only.
* ``libjmix_synth.so``: the seeded input generator (host C).
* ``libjmix_pipes.so``: the pipe-rate microbenchmarks (``pipe_rates.py``), kept
  out of libjmix.

Both are built in-tree under ``_build/`` so that they travel with the source.
"""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
INCLUDE = os.path.join(ROOT, "include")
LIBJMIX = os.path.join(BUILD, "libjmix.so")
LIBSYNTH = os.path.join(BUILD, "libjmix_synth.so")
LIBPIPES = os.path.join(BUILD, "libjmix_pipes.so")
PIPES_SRC = os.path.join(CSRC, "pipe_rates.cu")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def build_synth(force: bool = False) -> str:
    src = os.path.join(CSRC, "synth_gen.c")
    if force or _stale(LIBSYNTH, [src]):
        os.makedirs(BUILD, exist_ok=True)
        tmp = LIBSYNTH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-pthread", src, "-o", tmp, "-lm"])
        os.replace(tmp, LIBSYNTH)
    return LIBSYNTH


def jmix_sources():
    return sorted(p for p in glob.glob(os.path.join(CSRC, "*.cu")) if p != PIPES_SRC)


def jmix_deps():
    return (jmix_sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
            + sorted(glob.glob(os.path.join(INCLUDE, "*.h"))))


def build_libjmix(force: bool = False, verbose: bool = False) -> str:
    """nvcc -gencode arch=compute_100a,code=sm_100a ... -shared -> _build/libjmix.so.
    Each .cu compiles to an object in parallel, then one link."""
    srcs = jmix_sources()
    if not (force or _stale(LIBJMIX, jmix_deps())):
        return LIBJMIX
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    objs, procs = [], []
    for s in srcs:
        o = os.path.join(BUILD, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        cmd = [nvcc, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", s, "-o", o]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for cmd, p in procs:
        out, _ = p.communicate()
        if verbose or p.returncode:
            print(out.decode(errors="replace"))
        if p.returncode:
            failed.append(" ".join(cmd))
    if failed:
        raise RuntimeError("nvcc failed:\n" + "\n".join(failed))
    tmp = LIBJMIX + ".tmp%d" % os.getpid()
    cuda_lib = os.path.join(os.path.dirname(os.path.dirname(nvcc)), "lib64")
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-Xcompiler", "-fPIC", *objs, "-o", tmp,
                           "-Xlinker", "-rpath=" + cuda_lib])
    os.replace(tmp, LIBJMIX)
    return LIBJMIX


def build_pipes(force: bool = False) -> str:
    """nvcc ... -shared pipe_rates.cu -> _build/libjmix_pipes.so (sm_100a)."""
    if force or _stale(LIBPIPES, [PIPES_SRC]):
        os.makedirs(BUILD, exist_ok=True)
        tmp = LIBPIPES + ".tmp%d" % os.getpid()
        subprocess.check_call([_nvcc(), *NVCC_FLAGS, "-shared", PIPES_SRC, "-o", tmp])
        os.replace(tmp, LIBPIPES)
    return LIBPIPES


def build_all(force: bool = False) -> None:
    build_synth(force)
    build_libjmix(force)
    build_pipes(force)


if __name__ == "__main__":
    import sys
    build_synth(True)
    build_libjmix(True, verbose="-v" in sys.argv)
    print(LIBJMIX)

"""The C ABI from C: a small C99 program includes include/jmix.h (strict,
-Werror -pedantic), links against libjmix.so and calls the host-only entry
points (workspace sizes, schedules, validation); its answers must equal the
Python binding's.  No GPU is needed: none of these calls launches work."""
import os
import subprocess

import pytest

from mamba_selective_scan_jamba_b200 import build, jmix

PROGRAM = r"""
#include <stdio.h>
#include "jmix.h"

int main(void) {
  jm_dims d = {0};
  d.batch = 8; d.seqlen = 4096; d.d_inner = 8192; d.d_state = 16; d.d_conv = 4;
  d.dt_rank = 256; d.eps = 1e-6f; d.io = JM_BF16; d.discretization = JM_DISC_EULER;
  int parts = 0, two_pass = 0, bwd_parts = 0;
  if (jm_mixer_fwd_schedule(&d, &parts, &two_pass) != JM_OK) return 2;
  if (jm_scan_bwd_schedule(&d, &bwd_parts) != JM_OK) return 3;
  jm_dims step = d;
  step.seqlen = 1;  /* a decode step is one token per sequence */
  printf("%zu %zu %zu %d %d %d\n", jm_mixer_fwd_workspace_size(&d),
         jm_mixer_step_workspace_size(&step), jm_scan_bwd_workspace_size(&d), parts, two_pass,
         bwd_parts);
  d.d_state = 8;  /* not built: every size query says 0, a call says so too */
  printf("%zu %d\n", jm_mixer_fwd_workspace_size(&d),
         (int)jm_mixer_fwd_schedule(&d, &parts, &two_pass));
  printf("%s\n", jm_last_error() ? "message" : "none");
  return 0;
}
"""


def test_c_program_uses_the_abi(tmp_path):
    lib = build.build_libjmix()
    src = tmp_path / "use_jmix.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_jmix"
    libdir = os.path.dirname(lib)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", build.INCLUDE, str(src), "-o", str(exe), lib,
                           "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    first, second, third = out.stdout.split("\n")[:3]
    fws, sws, bws, parts, two_pass, bwd_parts = first.split()
    d = jmix.dims(8, 4096, 8192, 256)
    assert int(fws) == jmix.jm_mixer_fwd_workspace_size(d) > 0
    assert int(sws) == jmix.jm_mixer_step_workspace_size(jmix.dims(8, 1, 8192, 256)) > 0
    assert int(bws) == jmix.jm_scan_bwd_workspace_size(d) > 0
    assert (int(parts), bool(int(two_pass))) == jmix.jm_mixer_fwd_schedule(d)
    assert int(bwd_parts) == jmix.jm_scan_bwd_schedule(d)
    size0, status = second.split()
    assert int(size0) == 0 and int(status) == jmix.JM_ERR_UNSUPPORTED
    assert third == "message"


@pytest.mark.parametrize("std", ["-std=c99", "-std=c11"])
def test_header_is_plain_c(tmp_path, std):
    src = tmp_path / "h.c"
    src.write_text('#include "jmix.h"\nint main(void) { return 0; }\n')
    subprocess.check_call(["gcc", std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only",
                           "-I", build.INCLUDE, str(src)])

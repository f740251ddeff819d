"""The C ABI from C: include/gbs.h compiles as C99, a C program links against the
in-tree libgbs.so and calls entry points that need no GPU (version, status text,
workspace sizes, argument validation)."""
import os
import shutil
import subprocess

import pytest

from gated_block_sparse_gate_b200.build import INCLUDE, LIB, build

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "gbs.h"

int main(void) {
  gbs_params p;
  memset(&p, 0, sizeof p);
  p.B = 1; p.Hq = 32; p.Hkv = 8; p.N = 8192; p.d = 128; p.block = 64;
  p.mode = GBS_TRAIN; p.dtype = GBS_BF16;
  size_t fwd = gbs_workspace_bytes(&p, GBS_OP_FWD);
  size_t bwd = gbs_workspace_bytes(&p, GBS_OP_BWD);
  p.mode = GBS_THRESHOLD; p.topk = 16; p.tau = 0.05f;
  size_t thr = gbs_workspace_bytes(&p, GBS_OP_FWD);
  p.tau = 2.0f;  /* outside (0, 1] */
  gbs_status s = gbs_fwd(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  printf("%d %zu %zu %zu %d %s|%s\n", gbs_version(), fwd, bwd, thr, (int)s,
         gbs_status_string(s), gbs_last_error());
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_links_and_calls_the_abi(tmp_path):
    build()
    src = tmp_path / "use_gbs.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_gbs"
    libdir = os.path.dirname(LIB)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", INCLUDE, str(src), "-o", str(exe),
                    libdir + "/libgbs.so", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    version, fwd, bwd, thr, status = (int(v) for v in out[:5])
    assert version == (0 << 16) | 1
    assert 0 < fwd < thr and bwd > fwd
    assert status == 1 and "tau" in " ".join(out[5:])

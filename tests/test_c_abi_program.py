"""The boundary as a C or C++ user sees it: include/qsa.h compiles under strict
C99 and C++17, and a program linked against the in-tree library calls its
host-side entry points (size queries, argument checks, status strings) with no
GPU present."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "token_indexed_sparse_b200")

PROGRAM = r"""
#include <stdio.h>
#include "qsa.h"
int main(void) {
  int bad = 0;
  const size_t fw = qsa_forward_workspace_size(256, 256, 12, 1, 64);
  const size_t bw = qsa_backward_workspace_size(256, 256, 12, 1, 64);
  bad |= !(fw > 0 && bw > fw && fw % 256 == 0);
  bad |= qsa_forward_workspace_size(16, 16, 8, 1, 4) != 0;                 /* 8 heads per KV head */
  /* argument checks return before any CUDA work */
  bad |= qsa_forward(NULL, NULL, NULL, NULL, 16, 16, 12, 1, 4, 0.0625f, NULL, NULL, NULL, 0, NULL) !=
         QSA_ERR_INVALID_ARGUMENT;
  bad |= qsa_launch_count(256, 256, 12, 1, 64, 0) != QSA_FORWARD_STAGES;
  printf("%s|%s|%d\n", qsa_version(), qsa_status_string(QSA_ERR_MISALIGNED), qsa_launch_count(256, 256, 12, 1, 64, 1));
  return bad;
}
"""


@pytest.fixture(scope="module")
def lib_built():
    from token_indexed_sparse_b200 import build
    build.build()
    return os.path.join(LIBDIR, "libqsa_b200.so")


@pytest.mark.parametrize("compiler,flags,suffix", [("gcc", ["-std=c99"], ".c"), ("g++", ["-std=c++17"], ".cpp")])
def test_program_against_the_library(lib_built, tmp_path, compiler, flags, suffix):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    src = tmp_path / f"prog{suffix}"
    src.write_text(PROGRAM)
    exe = tmp_path / "prog"
    cmd = [compiler, *flags, "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-L", LIBDIR, "-lqsa_b200", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.stdout, r.stderr)
    version, status, launches = r.stdout.strip().split("|")
    assert "sm_100a" in version and status == "QSA_ERR_MISALIGNED" and int(launches) == 7

"""The boundary is a C ABI: a plain C99 program (strict, warnings as errors) includes the header,
links the shared library and calls its host-side entry points; the header also compiles as C++."""

import os
import shutil
import subprocess

import pytest

from block_sparse_long_dual_b200 import build as sfa_build
from block_sparse_long_dual_b200 import sfa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "block_sparse_long_dual_b200")

PROGRAM = r"""
#include <stdio.h>
#include "sfa.h"

int main(void) {
  sfa_shape ok = {1, 32, 8, 131072, 128, SFA_BF16};
  sfa_shape bad = {1, 32, 8, 1000, 128, SFA_BF16};   /* L not a multiple of the block */
  size_t off[4];
  const sfa_status st = sfa_workspace_layout(&ok, 128, off);
  printf("%d|%s|%zu|%d|%zu|%d|%zu\n", sfa_version(), sfa_status_string(SFA_ERR_SHAPE),
         sfa_block_scores_workspace(&ok, 128), (int)st, off[3],
         (int)sfa_workspace_layout(&bad, 128, off), sfa_block_scores_workspace(&bad, 128));
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib():
    sfa_build.build()
    return sfa.load()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_program_links_and_calls_the_library(lib, tmp_path):
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    cc = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE, str(src),
          "-L", PKG, "-lsfa", f"-Wl,-rpath,{PKG}", "-o", str(exe)]
    r = subprocess.run(cc, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    version, text, ws, st, off3, st_bad, ws_bad = r.stdout.strip().split("|")
    assert int(version) == lib.sfa_version()
    assert text == "invalid shape"
    nb, d = 131072 // 128, 128
    qbar = 32 * nb * d * 8
    assert int(ws) > qbar and int(st) == 0 and 0 < int(off3) < int(ws)
    assert int(st_bad) == 2 and int(ws_bad) == 0   # SFA_ERR_SHAPE, no workspace for an invalid shape


@pytest.mark.skipif(shutil.which("g++") is None, reason="no C++ compiler")
def test_header_compiles_as_cpp(tmp_path):
    src = tmp_path / "consumer.cpp"
    src.write_text('#include "sfa.h"\nint main() { return sfa_version() > 0 ? 0 : 1; }\n')
    r = subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE, "-c",
                        str(src), "-o", str(tmp_path / "consumer.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr

"""The C ABI from plain C: a C99 program that includes only include/lq.h
compiles without warnings (-Wall -Wextra -pedantic), links against liblq.so
and calls entry points that need no GPU (version, status strings, argument
checks, dispatch-table lookups).  The header also compiles as C++.  CPU only."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(ROOT, "quantized_linear_gemm_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "lq.h"

int main(void) {
  lq_variant v;
  lq_status s;
  memset(&v, 0, sizeof v);
  printf("version %s\n", lq_version());
  printf("status %s\n", lq_status_string(LQ_ERR_ALIGNMENT));
  s = lq_scaled_mm(LQ_FP8_DYNAMIC, NULL, NULL, NULL, NULL, NULL, 4, 128, 128, NULL, NULL);
  printf("null_C %d\n", (int)s);
  s = lq_select_variant(LQ_FP8_DYNAMIC, 8, 4096, 4096, &v);
  printf("select %d %d %d %d\n", (int)s, v.swap_ab, v.split_k, v.tile_n);
  printf("entries %lld\n", (long long)lq_dispatch_table_size());
  return 0;
}
"""


@pytest.fixture(scope="module")
def gcc():
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    return cc


def test_c99_program_uses_the_abi(gcc, tmp_path):
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I" + INCLUDE, str(src),
                        "-L" + LIBDIR, "-llq", "-Wl,-rpath," + LIBDIR, "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    lines = dict(line.split(" ", 1) for line in out.stdout.strip().splitlines())
    assert lines["version"].startswith("lq ")
    assert lines["status"] == "LQ_ERR_ALIGNMENT"
    assert int(lines["null_C"]) == 1                     # LQ_ERR_INVALID_ARG, nothing launched
    sel = [int(t) for t in lines["select"].split()]
    assert sel[0] == 0 and sel[1] in (0, 1) and sel[2] >= 1 and sel[3] in (16, 32, 64, 128, 256)
    assert int(lines["entries"]) > 0


def test_header_compiles_as_cpp(tmp_path):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no C++ compiler")
    src = tmp_path / "h.cpp"
    src.write_text('#include "lq.h"\nint main() { return LQ_OK; }\n')
    r = subprocess.run([gxx, "-std=c++17", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-I" + INCLUDE, str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr

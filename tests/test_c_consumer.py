"""include/e4b.h is a plain C header: a C99 program (and a C++ one) compiles against it with every
warning an error, links libe4b.so and calls the host-only entry points (CPU only).

The ctypes tests check the exports; this checks what a C caller sees: the header's types and
prototypes compile as C, the enum values and struct layouts are what the binding assumes, and
argument checks return their statuses through a plain C call.
"""

import ctypes
import os
import shutil
import subprocess

import pytest

from grouped_nf4_expert_b200 import build as e4b_build
from grouped_nf4_expert_b200 import e4b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "grouped_nf4_expert_b200")

PROGRAM = r"""
#include "e4b.h"
#include <stdio.h>
#include <string.h>

#define CHECK(c) do { if (!(c)) { printf("FAIL %s:%d %s\n", __FILE__, __LINE__, #c); return 1; } } while (0)

int main(void) {
  e4b_moe_dims d;
  e4b_sizes s;
  float lv[16];
  e4b_routing routing;
  memset(&d, 0, sizeof d);
  d.E = 128; d.H = 2048; d.I = 768; d.top_k = 8; d.r = 64; d.alpha = 128.0f;
  d.blocksize = 64; d.act = E4B_ACT_SILU_GLU;
  CHECK(e4b_get_sizes(&d, 8192, &s) == E4B_OK);
  CHECK(s.slots == 65536);
  CHECK(s.rows_cap % E4B_ROW_ALIGN == 0 && s.rows_cap >= 65536 + 128 * (E4B_ROW_ALIGN - 1));
  CHECK(s.workspace_bytes >= 256);
  d.r = 12;
  CHECK(e4b_get_sizes(&d, 8192, &s) == E4B_ERR_UNSUPPORTED);
  d.r = 64;
  CHECK(e4b_get_sizes(&d, -1, &s) == E4B_ERR_INVALID_ARG);
  CHECK(e4b_get_sizes(NULL, 1, &s) == E4B_ERR_INVALID_ARG);
  e4b_nf4_levels(lv);
  CHECK(lv[0] == -1.0f && lv[7] == 0.0f && lv[15] == 1.0f);
  CHECK(strncmp(e4b_status_string(E4B_ERR_WORKSPACE_TOO_SMALL), "E4B_ERR_WORKSPACE_TOO_SMALL", 27) == 0);
  CHECK(strstr(e4b_version(), "e4b") != NULL);
  memset(&routing, 0, sizeof routing);
  /* host-side validation: refused before any CUDA call */
  CHECK(e4b_route_permute(&d, 32, NULL, NULL, &routing, NULL, NULL, 0, NULL) == E4B_ERR_INVALID_ARG);
  CHECK(e4b_route_permute(&d, 0, NULL, NULL, NULL, NULL, NULL, 0, NULL) == E4B_OK);
  CHECK(e4b_nf4_quantize(NULL, 63, NULL, NULL, NULL) == E4B_ERR_INVALID_ARG);
  CHECK(e4b_profiler_enable(0) == E4B_OK);
  /* layouts the ctypes binding mirrors */
  CHECK(sizeof(e4b_moe_dims) == 32 && sizeof(e4b_nf4_experts) == 4 * sizeof(void *));
  CHECK(sizeof(e4b_routing) == 7 * sizeof(void *) && sizeof(e4b_fwd_buffers) == 6 * sizeof(void *));
  CHECK(sizeof(e4b_bwd_buffers) == 5 * sizeof(void *) && sizeof(e4b_sizes) == 32);
  CHECK(sizeof(e4b_kernel_time) == 64);
  printf("SIZES %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(e4b_moe_dims), sizeof(e4b_nf4_experts),
         sizeof(e4b_lora), sizeof(e4b_routing), sizeof(e4b_fwd_buffers), sizeof(e4b_bwd_buffers),
         sizeof(e4b_sizes), sizeof(e4b_kernel_time));
  printf("OK\n");
  return 0;
}
"""


def _compile_and_run(tmp_path, compiler, std, ext):
    exe = shutil.which(compiler)
    if exe is None:
        pytest.skip("%s not installed" % compiler)
    src = tmp_path / ("consumer" + ext)
    src.write_text(PROGRAM)
    out = tmp_path / ("consumer_" + compiler.replace("+", "x"))
    cmd = [exe, "-std=" + std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE, str(src),
           "-L", PKG, "-le4b", "-Wl,-rpath," + PKG, "-o", str(out)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(out)], capture_output=True, text=True, timeout=120)
    lines = r.stdout.split("\n")
    assert r.returncode == 0 and lines[-2] == "OK", r.stdout + r.stderr
    # the ctypes binding lays the structs out as the C compiler does
    sizes = [int(v) for v in lines[-3].split()[1:]]
    classes = [e4b.MoeDims, e4b.Nf4Experts, e4b.Lora, e4b.Routing, e4b.FwdBuffers, e4b.BwdBuffers, e4b.Sizes,
               e4b.KernelTime]
    assert sizes == [ctypes.sizeof(c) for c in classes]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    e4b_build.build()


def test_c99_program_compiles_links_and_runs(tmp_path):
    _compile_and_run(tmp_path, "gcc", "c99", ".c")


def test_cxx_program_compiles_links_and_runs(tmp_path):
    _compile_and_run(tmp_path, "g++", "c++11", ".cpp")

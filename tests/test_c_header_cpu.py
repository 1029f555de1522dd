"""CPU: include/rn.h is a plain C header and librn.so serves a C program.

A small C99 program (compiled with -Wall -Wextra -pedantic -Werror) includes
the header, links the library and calls it in validate-only mode, where the
argument checks run and nothing touches CUDA (the fake device addresses are
never dereferenced).  The same source also has to compile as C++, through the
header's extern "C" guard.
"""
import os
import shutil
import subprocess

import pytest

import rollout_parity_b200 as rn
from rollout_parity_b200 import build as rn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.dirname(rn.LIB_PATH)

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "rn.h"

#define EXPECT(cond)                                                   \
  do {                                                                 \
    if (!(cond)) {                                                     \
      fprintf(stderr, "line %d: %s\n", __LINE__, #cond);               \
      return 1;                                                        \
    }                                                                  \
  } while (0)

/* fake, 16-byte aligned device addresses 4 GiB apart (never dereferenced) */
static void* dev(int i) { return (void*)(uintptr_t)((1ull << 40) + ((uint64_t)i << 32)); }

int main(void) {
  const int64_t rows = 262144;
  const int32_t width = 128;
  const size_t ws = norm_bwd_workspace_bytes(rows, width);
  const char* d;
  /* (ceil(rows/32) + ceil(rows/256)) partial rows of width fp32 */
  EXPECT(ws == (size_t)(8192 + 1024) * 128 * 4);
  EXPECT(norm_bwd_workspace_bytes(rows, 12) == 0);

  rn_test_set_validate_only(1);
  EXPECT(gated_norm_fwd(rows, width, 1e-6f, RN_BF16, dev(0), dev(1), (const float*)dev(2),
                        dev(3), (float*)dev(4), NULL) == RN_OK);
  EXPECT(gated_norm_bwd(rows, width, 1e-6f, RN_BF16, dev(0), dev(1), (const float*)dev(2),
                        dev(3), (const float*)dev(4), dev(5), dev(6), (float*)dev(7), dev(8),
                        ws, NULL) == RN_OK);
  EXPECT(gated_norm_bwd(rows, width, 1e-6f, RN_BF16, dev(0), dev(1), (const float*)dev(2),
                        dev(3), (const float*)dev(4), dev(5), dev(6), (float*)dev(7), dev(8),
                        ws - 1, NULL) == RN_E_WORKSPACE);
  EXPECT(norm_fwd(rows, 12, 1e-6f, RN_BF16, dev(0), (const float*)dev(2), dev(3), NULL, NULL)
         == RN_E_WIDTH);
  EXPECT(norm_fwd(rows, width, 1e-6f, (rn_dtype)7, dev(0), (const float*)dev(2), dev(3), NULL,
                  NULL) == RN_E_DTYPE);
  EXPECT(norm_fwd(rows, width, 1e-6f, RN_F32, (const char*)dev(0) + 4, (const float*)dev(2),
                  dev(3), NULL, NULL) == RN_E_ALIGN);
  EXPECT(norm_fwd(rows, width, -1.0f, RN_F32, dev(0), (const float*)dev(2), dev(3), NULL, NULL)
         == RN_E_ARG);
  EXPECT(rmsnorm_fwd(rows, width, 1e-6f, 1.0f, RN_ACT_SIGMOID, RN_F16, dev(0), dev(1),
                     (const float*)dev(2), dev(3), (float*)dev(4), NULL) == RN_OK);
  EXPECT(rmsnorm_fwd(rows, width, 1e-6f, 1.0f, RN_ACT_NONE, RN_F16, dev(0), dev(1),
                     (const float*)dev(2), dev(3), (float*)dev(4), NULL) == RN_E_ARG);
  /* an output overlapping an input */
  EXPECT(norm_fwd(rows, width, 1e-6f, RN_BF16, dev(0), (const float*)dev(2), dev(0), NULL, NULL)
         == RN_E_ARG);
  rn_test_set_validate_only(0);

  d = rn_describe(width, RN_BF16);
  EXPECT(strstr(d, "acc=fp32") != NULL && strstr(d, "atomics=none") != NULL);
  EXPECT(strcmp(rn_describe(12, RN_BF16), "unsupported") == 0);
  EXPECT(strcmp(rn_status_string(RN_OK), "ok") == 0);
  EXPECT(rn_bwd_launches(rows, width, RN_BF16) >= 1);
  EXPECT(rn_test_set_geometry(-1, 0, 0) == RN_E_ARG);
  EXPECT(rn_test_set_geometry(0, 0, 0) == RN_OK);
  puts("c abi ok");
  return 0;
}
"""


@pytest.fixture(scope="module")
def built():
    rn_build.build()
    return rn.LIB_PATH


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_compiles_links_and_runs(built, tmp_path):
    src = tmp_path / "use_rn.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_rn"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    f"-I{INCLUDE}", str(src), f"-L{PKG}", "-lrn", f"-Wl,-rpath,{PKG}",
                    "-o", str(exe)], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "c abi ok"


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not installed")
def test_header_compiles_as_cpp(tmp_path):
    src = tmp_path / "use_rn.cpp"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", f"-I{INCLUDE}",
                    "-fsyntax-only", str(src)], check=True, capture_output=True, text=True)

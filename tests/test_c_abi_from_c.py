"""The C ABI used from plain C, without Python in between.

include/convrot.h must compile as strict C99 (and as C++), and a C program
linked against libconvrot.so must get the documented host-side answers. No GPU
is needed: the program makes only calls that return before any CUDA work
(version, status strings, workspace sizes, argument checks, the empty batch).
"""

from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "w8a8_rotated_int8_token_b200")

PROGRAM = r"""
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "convrot.h"

static int fails = 0;
#define CHECK(c)                          \
  do {                                    \
    if (!(c)) {                           \
      printf("FAIL line %d: %s\n", __LINE__, #c); \
      ++fails;                            \
    }                                     \
  } while (0)

int main(void) {
  void* fake = (void*)(uintptr_t)0x10000; /* aligned, never dereferenced: every call below returns on the host */
  size_t need = convrot_linear_workspace_bytes(4608, 9216, 3072, 256);
  CHECK(convrot_abi_version() == 9);
  CHECK(strcmp(convrot_status_string(CONVROT_OK), "ok") == 0);
  CHECK(strcmp(convrot_status_string(99), "unknown status") == 0);
  CHECK(need >= (size_t)4608 * 3072 + 4 * 4608);
  CHECK(convrot_linear_workspace_bytes(4608, 9216, 3072, 64) == 0);
  CHECK(convrot_linear_launch_count(4608, 9216, 3072, 256) == 2);
  CHECK(convrot_linear_launch_count(0, 9216, 3072, 256) == 0);
  CHECK(convrot_gemm_workspace_bytes() == 256);
  /* argument checks */
  CHECK(convrot_linear(fake, 64, 300, 256, fake, fake, 256, NULL, fake, fake, need, NULL) == CONVROT_ERR_INVALID_ARG);
  CHECK(convrot_linear(fake, 64, 256, 64, fake, fake, 256, NULL, fake, fake, need, NULL) == CONVROT_ERR_UNSUPPORTED);
  CHECK(convrot_linear(fake, 64, 256, 256, fake, fake, 256, NULL, fake, NULL, need, NULL) == CONVROT_ERR_WORKSPACE);
  CHECK(convrot_quant_act(NULL, 8, 256, 256, fake, fake, NULL) == CONVROT_ERR_INVALID_ARG);
  CHECK(convrot_linear_ex(fake, CONVROT_DTYPE_F16, 64, 256, 0, 256, fake, fake, CONVROT_WSCALE_CHANNEL, 256, NULL,
                          NULL, 7, fake, 0, fake, need, NULL) == CONVROT_ERR_UNSUPPORTED);
  /* an empty batch: nothing to do, nothing launched */
  CHECK(convrot_linear(NULL, 0, 3072, 256, fake, fake, 9216, NULL, NULL, NULL, 0, NULL) == CONVROT_OK);
  CHECK(convrot_quant_act(NULL, 0, 256, 256, NULL, NULL, NULL) == CONVROT_OK);
  CHECK(convrot_gemm_s32(NULL, fake, 0, 8, 256, NULL, NULL, 0, NULL) == CONVROT_OK);
  printf("%s\n", fails ? "failed" : "ok");
  return fails != 0;
}
"""


def _lib_path():
    path = os.path.join(PKG, "libconvrot.so")
    if not os.path.exists(path):
        pytest.skip("libconvrot.so is not built")
    return path


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_strict_c_and_links(tmp_path):
    _lib_path()
    src = tmp_path / "abi_check.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi_check"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE, str(src),
                         "-L", PKG, "-lconvrot", f"-Wl,-rpath,{PKG}", "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip().endswith("ok"), run.stdout + run.stderr


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_header_compiles_as_cxx(tmp_path):
    src = tmp_path / "abi_check.cc"
    src.write_text('#include "convrot.h"\nint main() { return convrot_abi_version() > 0 ? 0 : 1; }\n')
    cc = subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only", "-I",
                         INCLUDE, str(src)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr

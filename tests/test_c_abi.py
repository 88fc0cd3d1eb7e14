"""The boundary is plain C: a C99 program compiled with gcc -pedantic against include/owq.h
links libowq_b200.so and gets the documented answers from the calls that need no GPU
(version, status strings, handle and argument validation)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "weight_only_mixed_owq_b200")

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "owq.h"

static int fails = 0;
#define EXPECT(cond) do { if (!(cond)) { printf("FAIL line %d: %s\n", __LINE__, #cond); ++fails; } } while (0)

int main(void) {
  const uint16_t* h16 = (const uint16_t*)0x10000;
  uint16_t* o16 = (uint16_t*)0x10000;
  owq_layer_t none = NULL;
  owq_layer_t out = NULL;
  int s;
  EXPECT(strcmp(owq_version(), "") != 0);
  for (s = OWQ_OK; s <= OWQ_ERR_ARG; ++s) EXPECT(strncmp(owq_status_string(s), "OWQ_", 4) == 0);
  /* a handle that is not a live layer */
  EXPECT(owq_gemv(none, h16, o16, 1, NULL) == OWQ_ERR_HANDLE);
  EXPECT(owq_gemm(none, h16, o16, 64, NULL) == OWQ_ERR_HANDLE);
  EXPECT(owq_weak_grad(none, h16, h16, (float*)0x10000, 1, NULL) == OWQ_ERR_HANDLE);
  EXPECT(owq_input_grad(none, h16, o16, 1, NULL) == OWQ_ERR_HANDLE);
  EXPECT(owq_dequant(none, o16, NULL, NULL) == OWQ_ERR_HANDLE);
  EXPECT(owq_layer_free(NULL) == OWQ_OK);
  /* argument validation before any device use */
  EXPECT(owq_quantize(NULL, h16, 16, 128, 8, 3, 128, 1, (uint8_t*)0x10000, o16, o16,
                      (int32_t*)0x10000, o16, NULL) == OWQ_ERR_NULL);
  EXPECT(owq_quantize(h16, h16, 16, 128, 8, 5, 128, 1, (uint8_t*)0x10000, o16, o16,
                      (int32_t*)0x10000, o16, NULL) == OWQ_ERR_BITS);
  EXPECT(owq_quantize_noalloc(h16, h16, 16, OWQ_NOALLOC_MAX_K + 128, 8, 3, OWQ_NOALLOC_MAX_K + 128, 1,
                              (uint8_t*)0x10000, o16, o16, (int32_t*)0x10000, o16, NULL) == OWQ_ERR_SHAPE);
  EXPECT(owq_pack(NULL, 16, 128, 3, 128, h16, h16, (const int32_t*)0x10000, 1, h16, NULL, &out) == OWQ_ERR_NULL);
  EXPECT(out == NULL);
  EXPECT(owq_debug_inject(3, 1000) == OWQ_ERR_ARG);
  printf("fails=%d\n", fails);
  return fails;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_gets_documented_answers(tmp_path):
    from weight_only_mixed_owq_b200 import build
    lib = build.build()   # no-op when the library is up to date
    assert os.path.exists(lib)
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-L", LIBDIR, "-lowq_b200",
                         "-Wl,-rpath," + LIBDIR, "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "fails=0" in run.stdout

"""The C ABI from a plain C program (no Python, no C++), on the CPU.

The boundary is meant for callers in any language, so the header must
compile as ISO C99 (and as C++11) with warnings as errors, and a C program
linked against the in-tree libfa_b200.so must be able to call it. The program
below uses only the entry points that never reach a device: the status and
error strings, the backward workspace size, and argument validation, which
every compute entry point performs before any CUDA call.
"""

import os
import shutil
import subprocess

import pytest

import exact_attention_151_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")

PROGRAM = r"""
#include <stdio.h>
#include <stdint.h>
#include <stddef.h>
#include "fa.h"

int main(void) {
  size_t bytes = 0;
  int bad = 0;
  /* every status has a message */
  for (int s = 0; s <= 16; ++s) {
    const char* m = fa_status_string((fa_status)s);
    if (m == NULL || m[0] == '\0') bad |= 1;
  }
  /* backward workspace: two fp32 [B*H, 384] arrays (256-byte rounded) + 256 bytes */
  if (fa_bwd_workspace_size(2, 300, 3, &bytes) != FA_OK || bytes != (size_t)(2 * (2 * 3 * 384 * 4) + 256)) bad |= 2;
  if (fa_bwd_workspace_size(-1, 5, 5, &bytes) != FA_ERR_INVALID_ARG) bad |= 4;
  /* validation happens before any device call: null pointers, bad sizes, dtypes, head dims */
  if (fa_fwd(NULL, NULL, NULL, NULL, NULL, 1, 128, 2, 64, 0.125f, 0, FA_BF16, NULL) != FA_ERR_INVALID_ARG) bad |= 8;
  if (fa_fwd(NULL, NULL, NULL, NULL, NULL, -1, 128, 2, 64, 0.125f, 0, FA_BF16, NULL) != FA_ERR_INVALID_ARG) bad |= 16;
  if (fa_fwd((void*)256, (void*)256, (void*)256, (void*)256, (float*)256, 1, 128, 2, 96, 0.125f, 0, FA_BF16, NULL)
      != FA_ERR_UNSUPPORTED) bad |= 32;
  if (fa_fwd((void*)256, (void*)256, (void*)256, (void*)256, (float*)256, 1, 128, 2, 64, 0.125f, 0, (fa_dtype)7, NULL)
      != FA_ERR_INVALID_ARG) bad |= 64;
  if (fa_fwd((void*)264, (void*)256, (void*)256, (void*)256, (float*)256, 1, 128, 2, 64, 0.125f, 0, FA_BF16, NULL)
      != FA_ERR_MISALIGNED) bad |= 128;
  /* an empty problem is a no-op */
  if (fa_fwd(NULL, NULL, NULL, NULL, NULL, 0, 128, 2, 64, 0.125f, 0, FA_BF16, NULL) != FA_OK) bad |= 256;
  printf("%s %d\n", fa_status_string(FA_OK), bad);
  return bad != 0;
}
"""


def _compiler(name):
    path = shutil.which(name)
    if path is None:
        pytest.skip(f"{name} not available")
    return path


@pytest.mark.parametrize("lang,flags", [("c", ["-std=c99", "-pedantic"]), ("c++", ["-std=c++11"])])
def test_header_compiles_standalone(lang, flags, tmp_path):
    cc = _compiler("gcc" if lang == "c" else "g++")
    r = subprocess.run([cc, *flags, "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", lang,
                        os.path.join(INCLUDE, "fa.h")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_plain_c_program_links_and_calls_the_library(tmp_path):
    cc = _compiler("gcc")
    lib = fa.load_library()._name  # the in-tree shared object the binding loads
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", f"-I{INCLUDE}", str(src), lib,
                        f"-Wl,-rpath,{os.path.dirname(lib)}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.stdout, run.stderr)
    assert run.stdout.strip().endswith(" 0")

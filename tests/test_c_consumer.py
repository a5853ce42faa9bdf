"""The boundary from plain C (no Python, no torch): a C99 program compiled
against include/fg8.h and linked with libfg8.so calls the library, checks
its version and status strings, gets argument errors back before any device
is touched, and, on this GPU-less host, FG8_ERR_UNSUPPORTED_DEVICE for a
well-formed call (no CPU fallback)."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <stdint.h>
#include "fg8.h"

int main(void) {
  int bad = 0;
  if (fg8_version() <= 0) bad |= 1;
  if (fg8_status_string(FG8_OK) == NULL || fg8_status_string(FG8_ERR_TIMEOUT) == NULL) bad |= 2;
  /* shape and format errors come back before any device is looked up */
  uintptr_t p = (uintptr_t)1 << 24;   /* aligned, never dereferenced */
  void* a = (void*)p;
  if (fg8_quantize_act(a, 4, 256, 256, a, a, (fg8_scale_fmt)2, NULL) != FG8_ERR_INVALID_ARG) bad |= 4;
  if (fg8_quantize_act(a, 4, 120, 128, a, a, FG8_SCALE_FLOAT, NULL) != FG8_ERR_ALIGNMENT) bad |= 8;
  if (fg8_linear(a, 16, 256, 256, 256, a, a, NULL, a, 256, FG8_SCALE_FLOAT, a, 1, NULL) != FG8_ERR_WORKSPACE)
    bad |= 16;
  if (fg8_linear_workspace_bytes(16, 256, 256, FG8_SCALE_UE8M0) == 0) bad |= 32;
  if (fg8_linear(a, 0, 256, 256, 256, a, a, NULL, a, 256, FG8_SCALE_FLOAT, a, 0, NULL) != FG8_OK) bad |= 64;
  /* a well-formed call needs a B200 */
  fg8_status st = fg8_quantize_act(a, 4, 256, 256, a, a, FG8_SCALE_UE8M0, NULL);
  printf("%d %d %s\n", bad, (int)st, fg8_status_string(st));
  return bad;
}
"""


def test_c_program_links_and_calls_the_library(tmp_path):
    import torch
    if torch.cuda.is_available():
        pytest.skip("with a GPU present, the well-formed call would launch")
    import fine_grained_fp8_act_b200 as fg8
    lib = fg8.library_path()
    src = tmp_path / "use_fg8.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_fg8"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    lib, "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    bad, st, _ = r.stdout.split(" ", 2)
    assert bad == "0" and int(st) == 3  # FG8_ERR_UNSUPPORTED_DEVICE

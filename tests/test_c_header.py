"""The header is plain C: a C99 program that includes include/qlora.h compiles with gcc, links
against libqlora.so and calls the host-only entry points (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROG = r"""
#include <stdio.h>
#include <string.h>
#include "qlora.h"

int main(void) {
  qlora_weight_t w;
  memset(&w, 0, sizeof w);
  w.fmt = QLORA_FMT_NF4;
  w.N = 14336;
  w.K = 4096;
  w.codes = (const uint8_t*)0x100000;
  w.scales = (const void*)0x200000;
  size_t ws = qlora_workspace_size(QLORA_OP_BWD, &w, 4096, 64, 0);
  size_t bad = qlora_workspace_size(QLORA_OP_BWD, &w, 4096, 12, 0);
  size_t lq = qlora_loftq_workspace_size(14336, 4096, 64);
  qlora_status_t st = qlora_quantize(&w, (const void*)0x300004, 0, NULL);
  printf("%zu %zu %zu %d %s\n", ws, bad, lq, (int)st, qlora_status_string(QLORA_ERR_WORKSPACE));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c_and_links(tmp_path):
    from bit_quantized_base_b200 import build
    lib = build.build()
    src = tmp_path / "use_qlora.c"
    src.write_text(PROG)
    exe = tmp_path / "use_qlora"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-l:" + os.path.basename(lib),
                    "-Wl,-rpath," + libdir, "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    ws, bad, lq, st = int(out[0]), int(out[1]), int(out[2]), int(out[3])
    assert ws > 0 and bad == 0
    assert lq >= 4 * 14336 * 4096
    assert st == 1                               # QLORA_ERR_INVALID_ARG: v not 16-byte aligned
    assert " ".join(out[4:])

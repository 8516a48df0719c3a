"""The boundary is a C ABI: a C11 program that includes include/domino.h compiles with gcc, links
against libdomino.so and calls the host-only entry points (no GPU needed)."""
import os
import subprocess

import pytest

from draft_block_causal_b200 import build, domino

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "domino.h"

int main(void) {
  domino_shape_t s = {1, 16, 4096, 1024, 256, 151936, DOMINO_DTYPE_BF16};
  domino_shape_t bad = {1, 16, 4096, 1024, 256, 151937, DOMINO_DTYPE_BF16};
  domino_weights_t w = {0};
  printf("abi %d\n", (int)domino_abi_version());
  printf("ws %d %d\n", domino_workspace_bytes(&s) > 0, domino_workspace_bytes(&bad) == 0);
  printf("arena %d\n", domino_arena_bytes(&s) > 0);
  printf("reject %d\n", domino_draft_greedy(&s, &w, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) == DOMINO_ERR_INVALID_ARGUMENT);
  printf("status %s\n", domino_status_string(DOMINO_STATUS_BAD_TOKEN));
  return 0;
}
"""


def test_c_program_compiles_links_and_runs(tmp_path):
    build.build()
    src = tmp_path / "use_domino.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_domino"
    libdir = os.path.dirname(domino.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe), "-L", libdir, "-ldomino", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines()
    assert out[0] == "abi 2"
    assert out[1] == "ws 1 1"
    assert out[2] == "arena 1"
    assert out[3] == "reject 1"
    assert out[4].startswith("status ") and "token" in out[4]

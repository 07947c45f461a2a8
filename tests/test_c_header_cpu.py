"""The boundary is a plain C ABI: a C99 program that includes include/star_attn.h
compiles warning-free with -pedantic, links against libstarattn.so and calls it
(host-side calls only: version, workspace sizing, argument validation)."""
import os
import shutil
import subprocess

import pytest

import block_sparse_attention_phase_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SOURCE = r"""
#include <stdio.h>
#include "star_attn.h"
int main(void) {
  star_attn_shape_t s = {1, 32, 8, 128, 32768, 4096, 0.0f};
  printf("%s\n", star_attn_version());
  printf("%zu\n", star_attn_workspace_bytes(&s, STAR_PHASE2_DECODE, 1));
  printf("%d\n", (int)star_attn_phase1(&s, 0, 0, 0, 0, 0, 0));
  printf("%s\n", star_attn_status_string(STAR_ERR_CACHE_FULL));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_is_c99_and_library_links(tmp_path):
    sa.lib()  # built in-tree
    src = tmp_path / "main.c"
    src.write_text(SOURCE)
    exe = tmp_path / "main"
    libdir = os.path.dirname(sa.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
           os.path.join(ROOT, "include"), str(src), "-L", libdir, "-l:libstarattn.so",
           f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    assert out[0] == sa.version()
    shape = sa.make_shape(1, 32, 8, 128, 32768, 4096)
    assert int(out[1]) == sa.workspace_bytes(shape, sa.STAR_PHASE2_DECODE)
    assert out[2] == "1"  # STAR_ERR_INVALID_ARG: null pointers, nothing launched
    assert out[3] == "query-local cache full"

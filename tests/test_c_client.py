"""The boundary from plain C: a C11 program includes include/attn.h, links
libattn.so and calls the entry points on argument errors (which return before any
device work), so this runs without a GPU."""
import os
import subprocess

import pytest

from exact_attention_103_b200 import build as ea_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "attn.h"

int main(void) {
  void* p = (void*)0x10000;  /* never dereferenced: validation returns first */
  attn_status_t s = attn_fwd(p, p, p, p, (float*)p, 1, 1, 128, 96, 0, 0.1f, NULL, NULL);
  printf("%s\n", attn_status_string(s));
  printf("%s\n", attn_last_error());
  attn_fwd_opts_t opts;
  memset(&opts, 0, sizeof(opts));
  opts.rescale_threshold = 100.f;
  s = attn_fwd_ex(p, p, p, p, (float*)p, 1, 1, 128, 128, 0, 0.1f, NULL, &opts, NULL);
  printf("%s\n", attn_status_string(s));
  s = attn_fwd_e4m3(p, p, p, p, (float*)p, 1, 1, 128, 64, 0, 0.1f, 1.f, 1.f, 1.f, NULL, NULL, NULL);
  printf("%s\n", attn_status_string(s));
  attn_bwd_opts_t bo;
  memset(&bo, 0, sizeof(bo));
  s = attn_bwd_ex(p, p, p, p, (float*)p, p, p, p, p, 0, 1, 128, 128, 1, 0.1f, NULL, 1, NULL, 0,
                  &bo, NULL);
  printf("%s\n", attn_status_string(s));
  printf("%zu\n", attn_bwd_workspace_size(2, 16, 8192, 128, 16384, 1));
  return 0;
}
"""


def test_plain_c_program_uses_the_abi(tmp_path):
    lib = ea_build.build()
    src = tmp_path / "client.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "client"
    libdir = os.path.dirname(lib)
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe), "-L", libdir, "-lattn", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    lines = out.stdout.splitlines()
    assert lines[0] == "ATTN_ERR_UNSUPPORTED"
    assert "head dim" in lines[1]
    assert lines[2] == "ATTN_ERR_INVALID_ARG"
    assert lines[3] == "ATTN_ERR_UNSUPPORTED"
    assert lines[4] == "ATTN_OK"  # B = 0: nothing to do
    assert lines[5] == str(2 * 8192 * 16 * 4)

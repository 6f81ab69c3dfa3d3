"""The C ABI from plain C: a C99 program that includes include/gpt2attn.h and
links against the library compiles, links and runs. Only calls that need no
GPU are made (sizes, argument checks, status strings)."""

import os
import shutil
import subprocess

import pytest

from causal_self_attention_flashattention_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "gpt2attn.h"

int main(void) {
  size_t ws = 0, fused = 0, dec = 0;
  int st = gpt2_attn_bwd_workspace_size(16, 1024, 12, 64, &ws);
  st |= gpt2_attn_bwd_fused_workspace_size(16, 1024, 12, 64, &fused);
  st |= gpt2_attn_decode_workspace_size(2, 1000, 3, 64, &dec);
  /* Rejected before any CUDA call: D other than 64, a null pointer. */
  int unsup = gpt2_attn_fwd((const void*)0x10000, (void*)0x10000, (float*)0x10000,
                            1, 128, 12, 128, 0.125f, (gpt2attn_stream_t)0);
  int inval = gpt2_attn_fwd((const void*)0, (void*)0x10000, (float*)0x10000,
                            1, 128, 12, 64, 0.125f, (gpt2attn_stream_t)0);
  printf("%d %zu %zu %zu %d %d %d\n%s\n", st, ws, fused, dec, unsup, inval,
         gpt2_attn_version(), gpt2_attn_status_string(GA_ERR_ALIGNMENT));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c99_program_uses_the_abi(tmp_path):
    lib = ops.lib()._name
    src = tmp_path / "use_abi.c"
    exe = tmp_path / "use_abi"
    src.write_text(PROGRAM)
    libdir = os.path.dirname(lib)
    libname = os.path.basename(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, f"-l:{libname}", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True, text=True)
    lines = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    st, ws, fused, dec, unsup, inval, version = lines[0].split()
    align = lines[1]
    assert int(st) == ops.GA_OK
    assert int(ws) == ops.bwd_workspace_size(16, 1024, 12, 64)
    assert int(fused) == ops.bwd_fused_workspace_size(16, 1024, 12, 64)
    assert int(dec) == ops.decode_workspace_size(2, 1000, 3, 64)
    assert int(unsup) == ops.GA_ERR_UNSUPPORTED
    assert int(inval) == ops.GA_ERR_INVALID_ARG
    assert int(version) == ops.version()
    assert align == ops.status_string(ops.GA_ERR_ALIGNMENT)

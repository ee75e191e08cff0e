"""include/attn.h is a C header: a C99 program includes it, takes the address of every function it declares,
links against libattn.so and calls the host-only entry points (no GPU needed: argument errors are detected
before any CUDA call, and a well-formed call without a GPU must fail loudly)."""
import os
import shutil
import subprocess

import pytest
import torch

import causal_self_attention_bf16_b200 as attn
from causal_self_attention_bf16_b200 import build as attn_build
from test_abi import HEADER, declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "attn.h"

typedef void (*any_fn)(void);
static const any_fn every_declared[] = { %(functions)s };

int main(void) {
  size_t ws;
  int fails = 0;
  if (sizeof(every_declared) / sizeof(every_declared[0]) != %(count)d) return 10;
  if (attn_abi_version() != 2) return 11;
  if (strcmp(attn_status_string(ATTN_ERR_MISALIGNED), "ATTN_ERR_MISALIGNED") != 0) return 12;
  if (strcmp(attn_status_string((attn_status)99), "ATTN_ERR_UNKNOWN") != 0) return 13;
  ws = attn_bwd_workspace_bytes(2, 3, 100, 128);   /* 2 * 256-rounded (rows * 4) + rows * 512, rows = 768 */
  if (ws != 2 * 3072 + 768 * 512) return 14;
  if (attn_bwd_workspace_bytes(1, 1, 1, 64) != 0) return 15;
  /* argument errors: reported before any CUDA call */
  fails += attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 2, 128, 128, 0.088f, NULL) != ATTN_ERR_INVALID_ARG;
  fails += attn_qk_norm_rope(NULL, NULL, NULL, NULL, NULL, 1, 8, 2, 2, 128, 10000.f, 1e-6f,
                             ATTN_ROPE_INTERLEAVED, NULL) != ATTN_ERR_INVALID_ARG;
  fails += attn_decode_workspace_bytes(2, 8, 3, 1, 1000, 128) != 0;
  if (%(no_gpu)d) {
    /* a well-formed in-place prologue call on a machine without a GPU fails loudly */
    void* fake = (void*)(size_t)(1ull << 40);
    void* fake_k = (void*)(size_t)((1ull << 40) + (1ull << 24));
    fails += attn_qk_norm_rope(fake, fake_k, fake, fake_k, NULL, 1, 8, 2, 2, 128, 10000.f, 1e-6f, ATTN_ROPE_HALF,
                               NULL) != ATTN_ERR_CUDA;
  }
  if (fails) return 20 + fails;
  printf("c abi ok: %%d functions\n", (int)(sizeof(every_declared) / sizeof(every_declared[0])));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c99_and_links(tmp_path):
    lib = attn_build.build()
    names = declared_functions()
    src = PROGRAM % {"functions": ", ".join(f"(any_fn){n}" for n in names), "count": len(names),
                     "no_gpu": 0 if torch.cuda.is_available() else 1}
    c_file = tmp_path / "abi.c"
    c_file.write_text(src)
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER),
           str(c_file), "-o", str(exe), lib, f"-Wl,-rpath,{lib_dir}"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, f"exit {run.returncode}: {run.stdout}{run.stderr}"
    assert f"{len(names)} functions" in run.stdout
    assert set(names) == set(attn.SIGNATURES)

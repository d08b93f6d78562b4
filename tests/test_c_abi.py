"""The boundary is a C ABI: a plain C program (gcc, C11, no CUDA headers)
includes include/fa.h, links libfa.so and calls the host-side entry points
and argument checks, none of which touch a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <math.h>
#include <stdio.h>
#include <string.h>
#include "fa.h"

static int fails = 0;
#define CHECK(c) do { if (!(c)) { printf("FAIL line %d: %s\n", __LINE__, #c); ++fails; } } while (0)

int main(void) {
  CHECK(strcmp(fa_status_string(FA_OK), "ok") == 0);
  CHECK(fa_status_string((fa_status)99) != NULL);
  float lv[16];
  CHECK(fa_tq_codebook(128, 4, lv) == FA_OK);
  for (int i = 0; i < 16; ++i) CHECK(lv[i] == -lv[15 - i]);
  for (int i = 1; i < 16; ++i) CHECK(lv[i] > lv[i - 1]);
  CHECK(fabsf(lv[15] - 0.23677f) < 1e-4f);  /* the outermost 4-bit level at d = 128 */
  CHECK(fa_tq_codebook(127, 4, lv) == FA_ERR_INVALID);
  CHECK(fa_decode_workspace_size(16, 32, 32768, 128) > 0);
  CHECK(fa_tq_decode_workspace_size(2, 8, 128, 4096) == (size_t)2 * 8 * 2 * 130 * 4);

  fa_fwd_params p;
  memset(&p, 0, sizeof p);
  CHECK(fa_attention_fwd(NULL, NULL) == FA_ERR_INVALID);
  p.batch = 1; p.hq = 3; p.hkv = 2; p.head_dim = 128; p.seqlen_q = p.seqlen_k = 64;
  p.q_dtype = FA_BF16; p.kv_dtype = FA_BF16; p.softmax_scale = 0.125f;
  CHECK(fa_attention_fwd(&p, NULL) == FA_ERR_INVALID);  /* hq % hkv != 0 */
  p.hq = 4; p.head_dim = 288;  /* a multiple of 32 without a tensor-core kernel */
  CHECK(fa_attention_fwd(&p, NULL) == FA_ERR_UNSUPPORTED);
  p.head_dim = 128; p.seqlen_q = 0;
  CHECK(fa_attention_fwd(&p, NULL) == FA_OK);  /* nothing to do */

  fa_merge_params m;
  memset(&m, 0, sizeof m);
  m.rows = 4; m.head_dim = 48;
  CHECK(fa_attention_merge(&m, NULL) == FA_ERR_INVALID);
  CHECK(fa_attention_fwd_acc(&p, NULL, NULL, 4, NULL) == FA_ERR_INVALID);  /* unknown flag */

  fa_tq_compress_params c;
  memset(&c, 0, sizeof c);
  c.rows = 1; c.head_dim = 128; c.bits = 5; c.x_dtype = FA_BF16;
  CHECK(fa_tq_compress(&c, NULL) == FA_ERR_UNSUPPORTED);
  printf("%s\n", fails ? "failed" : "c abi ok");
  return fails != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_program_links_and_calls_the_library(tmp_path):
    from flashattention_attention_b200 import build
    lib = build.build()
    src = tmp_path / "abi.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi"
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", os.path.dirname(lib), "-lfa", "-lm", "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c abi ok" in r.stdout, r.stdout + r.stderr

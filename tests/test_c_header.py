"""The boundary is a C ABI: include/mla.h compiles as plain C (C99) and as C++, and
a C program links against the library and calls its host-only entry points (no
device work, so this runs without a GPU)."""

import os
import shutil
import subprocess

import pytest

from head_latent_attention_06_b200 import build as mla_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INC = os.path.join(ROOT, "include")

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "mla.h"

int main(void) {
  /* host-side argument checks only: nothing here reaches a CUDA launch */
  if (mla_absorb_q(0, 0, 0, 4, 0, 128, 512, 0) != MLA_ERR_INVALID_VALUE) return 1;
  if (mla_up_proj_v(0, 0, 0, 4, 128, 64, 512, 0) != MLA_ERR_UNSUPPORTED) return 2;
  mla_decode_args_t a;
  memset(&a, 0, sizeof a);
  a.B = 64; a.s_q = 1; a.H = 128; a.d_c = MLA_D_C; a.d_r = MLA_D_R; a.page_size = MLA_PAGE_SIZE;
  a.num_pages = 4096; a.max_pages_per_seq = 64; a.kv_dtype = MLA_KV_BF16; a.max_seq_len = 4096;
  a.softmax_scale = 0.0722f;
  int32_t splits = 0;
  if (mla_decode_num_splits(&a, &splits) != MLA_OK || splits != 1) return 3;
  size_t bytes = 0;
  if (mla_decode_workspace_size(&a, &bytes) != MLA_OK || bytes != 256) return 4;
  if (mla_decode_paged(&a, 0) != MLA_ERR_INVALID_VALUE) return 5;   /* no workspace */
  mla_write_kv_args_t w;
  memset(&w, 0, sizeof w);
  w.B = 64; w.s_q = 1; w.d_h = 7168; w.d_c = MLA_D_C; w.d_r = MLA_D_R; w.page_size = MLA_PAGE_SIZE;
  w.num_pages = 4096; w.max_pages_per_seq = 64; w.kv_dtype = MLA_KV_BF16; w.rope_base = 10000.f;
  if (mla_write_kv_workspace_size(&w, &bytes) != MLA_OK || bytes < 256) return 6;
  if (strcmp(mla_status_string(MLA_ERR_MISALIGNED), "MLA_ERR_MISALIGNED") != 0) return 7;
  mla_step_args_t s;
  memset(&s, 0, sizeof s);
  s.B = 64; s.s_q = 1; s.H = 128; s.d_c = MLA_D_C; s.d_r = MLA_D_R; s.page_size = MLA_PAGE_SIZE;
  s.num_pages = 4096; s.max_pages_per_seq = 64; s.kv_dtype = MLA_KV_Q4_0; s.max_seq_len = 4096;
  s.softmax_scale = 0.0722f; s.fuse = -1;
  /* one split: the decode's 256 bytes, the step's flags, q_lat and o_lat */
  if (mla_decode_step_workspace_size(&s, &bytes) != MLA_OK || bytes != 512 + 2 * 64 * 128 * 512 * 2) return 8;
  int32_t launches = 0;
  if (mla_decode_step_launches(&s, &launches) != MLA_OK || launches != 3) return 9;
  if (mla_decode_step(&s, 0) != MLA_ERR_INVALID_VALUE) return 10;     /* no workspace */
  if (mla_fold_hadamard(0, 0, 0, 0, 0, 0) != MLA_OK) return 11;       /* nothing to fold */
  printf("ok\n");
  return 0;
}
"""


def _cc():
    return shutil.which("gcc") or shutil.which("cc")


@pytest.mark.skipif(_cc() is None, reason="no C compiler")
@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++11")])
def test_header_compiles_standalone(tmp_path, lang, std):
    src = tmp_path / ("h." + ("c" if lang == "c" else "cpp"))
    src.write_text('#include "mla.h"\nint main(void) { return MLA_OK; }\n')
    cc = _cc() if lang == "c" else (shutil.which("g++") or _cc())
    r = subprocess.run([cc, std, "-Wall", "-Werror", "-pedantic", "-I", INC, "-fsyntax-only", str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


@pytest.mark.skipif(_cc() is None, reason="no C compiler")
def test_c_program_links_and_calls_host_entry_points(tmp_path):
    lib = mla_build.build()
    src = tmp_path / "prog.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "prog"
    libdir = os.path.dirname(lib)
    r = subprocess.run([_cc(), "-std=c99", "-I", INC, str(src), "-o", str(exe), lib,
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)

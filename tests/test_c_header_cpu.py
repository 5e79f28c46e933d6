"""The boundary is a plain C ABI: a C99 program that includes only
include/sa.h compiles with gcc, links against libsa.so and makes the
host-only calls (version, validation, workspace sizes, status strings)
without a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

sa = pytest.importorskip("top_block_sparse_b200.sa")

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "sa.h"

static sa_params decode_params(void) {
  sa_params p;
  memset(&p, 0, sizeof p);
  p.batch = 2; p.num_q_heads = 8; p.num_kv_heads = 2; p.head_dim = 128;
  p.ctx_len = 4096; p.kv_capacity = 4097; p.n_q = 1; p.block_size = 64;
  p.pool = SA_POOL_MEAN; p.pool_stride = 4; p.top_k = 8; p.dtype = SA_BF16;
  p.out_dtype = SA_BF16; p.select = SA_SEL_QUERY0; p.sink_keys = 64; p.window_keys = 128;
  return p;
}

int main(void) {
  sa_params p = decode_params();
  if (sizeof(sa_params) != 96) return 10;
  if (sa_version() != 103) return 11;
  if (sa_workspace_size(&p, SA_OP_DECODE) == 0) return 12;
  if (sa_workspace_size(&p, SA_OP_SCORE_TOPK) == 0) return 13;
  p.head_dim = 64;                                   /* not built */
  if (sa_workspace_size(&p, SA_OP_DECODE) != 0) return 14;
  if (sa_pool_keys(&p, NULL, NULL, NULL) != SA_ERR_UNSUPPORTED) return 15;
  if (strlen(sa_last_error()) == 0) return 16;
  p = decode_params();
  p.pool = SA_POOL_OVERLAP; p.pool_stride = 16; p.pool_kernel = 8;   /* l < s */
  if (sa_pool_keys(&p, NULL, NULL, NULL) != SA_ERR_INVALID) return 17;
  if (sa_pool_keys(NULL, NULL, NULL, NULL) != SA_ERR_INVALID) return 18;
  if (strcmp(sa_status_string(SA_OK), sa_status_string(SA_ERR_INDEX)) == 0) return 19;
  if (sa_append_kv(&p, NULL, NULL, NULL, NULL, NULL) != SA_ERR_INVALID) return 20;
  printf("ok %d\n", sa_version());
  return 0;
}
"""


def test_c99_program_uses_the_header_and_library(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(sa.lib_path())
    src = tmp_path / "abi_check.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi_check"
    build = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                            str(src), "-L", lib_dir, "-lsa", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert run.stdout.strip() == "ok 103"

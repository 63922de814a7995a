"""The boundary is a C ABI: a plain C99 program includes include/qsa.h (with
-Wall -Wextra -Werror), links libqsa.so and calls it. Only calls that need no
GPU are made: the version, the status strings, a workspace size, and a prefill
call whose NULL arguments host validation refuses before any launch."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_attention_17_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "qsa.h"

int main(void) {
  qsa_config c;
  memset(&c, 0, sizeof c);
  c.num_q_heads = 16; c.num_kv_heads = 2; c.head_dim = 128; c.idx_heads = 4; c.idx_dim = 64;
  c.block_size = 64; c.budget = 2048; c.dtype = QSA_BF16;
  size_t ws = qsa_prefill_workspace_size(&c, 1, 8192, 8192);
  qsa_status s = qsa_prefill(&c, 1, 8192, 8192, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                             NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  char msg[256];
  strncpy(msg, qsa_last_error(), sizeof msg - 1);
  msg[sizeof msg - 1] = 0;
  c.rope_dim = 6;   /* not a multiple of 4 */
  qsa_status s2 = qsa_prefill(&c, 1, 8192, 8192, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                              NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  qsa_set_keys_visited(NULL);
  printf("%d|%s|%s|%zu|%s\n", qsa_version(), qsa_status_string(s), msg, ws,
         qsa_status_string(s2));
  return s == QSA_ERR_INVALID_ARG && s2 == QSA_ERR_INVALID_ARG && ws > 0 ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_uses_the_library(tmp_path):
    lib = os.path.join(PKG, "libqsa.so")
    if not os.path.exists(lib):
        pytest.skip("libqsa.so is not built")
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", PKG, "-lqsa", f"-Wl,-rpath,{PKG}", "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    version, status, msg, ws, status2 = r.stdout.strip().split("|")
    assert int(version) >= 101
    assert status == "QSA_ERR_INVALID_ARG" and "NULL" in msg
    assert int(ws) > 0
    assert status2 == "QSA_ERR_INVALID_ARG"

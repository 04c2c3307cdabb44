"""The ABI is plain C: a C99 program includes include/qsa.h, links libqsa.so and calls the
entry points that need no GPU (sizing, argument checks)."""
import os
import shutil
import subprocess

import pytest

from sparse_attention_decode_02_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "qsa.h"

int main(void) {
  qsa_config c;
  memset(&c, 0, sizeof c);               /* zero fields take the defaults */
  c.n_layers = 12; c.max_ctx = 262144; c.d_idx = 128; c.n_idx_heads = 16; c.top_k_tokens = 2048;
  c.n_q_heads = 32; c.n_kv_heads = 4; c.head_dim = 128; c.rope_base = 10000.0f; c.rms_eps = 1e-6f;
  size_t kv = qsa_buffer_bytes(&c, QSA_BUF_KV);
  size_t cells = qsa_layer_bytes(&c, QSA_BUF_MAX_CELLS);
  c.kv_format = QSA_KV_FP8;
  size_t kv8 = qsa_buffer_bytes(&c, QSA_BUF_KV);
  size_t scales = qsa_buffer_bytes(&c, QSA_BUF_KV_SCALES);
  c.d_idx = 96;                          /* unsupported: sizes are 0 */
  size_t bad = qsa_buffer_bytes(&c, QSA_BUF_KV);
  qsa_ctx* ctx = NULL;
  qsa_status st = qsa_create(NULL, &ctx);
  int32_t status = 0;
  printf("%zu %zu %zu %zu %zu %d %d %d %s\n", kv, cells, kv8, scales, bad, (int)st, (int)qsa_n_ctx(NULL, 0),
         (int)qsa_get_device_status(NULL, &status), qsa_last_error(NULL));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_library_links(tmp_path):
    lib = qbuild.build()
    src = tmp_path / "use_qsa.c"
    src.write_text(_PROGRAM)
    exe = tmp_path / "use_qsa"
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           lib, f"-Wl,-rpath,{os.path.dirname(lib)}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    kv, cells, kv8, scales, bad, st, n, dst, msg = r.stdout.split(maxsplit=8)
    assert int(kv) == 262144 * 4 * 128 * 2 and int(cells) == 2051
    assert int(kv8) == int(kv) // 2 and int(scales) == 262144 * 4 * 2 * 4
    assert int(bad) == 0 and int(st) == 1 and int(n) == -1 and int(dst) == 1
    assert msg.strip() == "null context"

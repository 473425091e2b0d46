"""The C ABI from a plain C host: include/hstu.h compiles as C11 (gcc, no C++),
a C program links against the in-tree libhstu.so and runs its host-only
entry points (sizes, layouts, status strings, argument checks that return
before any launch).  No GPU is used."""
import os
import shutil
import subprocess
import tempfile

import pytest

from hstu_sequential_transducer_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "hstu.h"

#define CHECK(c) do { if (!(c)) { printf("failed: %s (line %d)\n", #c, __LINE__); return 1; } } while (0)

int main(void) {
  hstu_config c;
  memset(&c, 0, sizeof(c));
  c.d_model = 256; c.num_heads = 2; c.head_dim = 128;
  c.num_pos_buckets = 32; c.num_time_buckets = 32; c.max_seq_len = 8192;
  c.norm_N = 256.0f; c.ln_eps = 1e-5f; c.dtype = HSTU_BF16; c.io_dtype = HSTU_F32;

  CHECK(strncmp(hstu_version(), "hstu-b200", 9) == 0);
  CHECK(strcmp(hstu_status_string(HSTU_OK), "ok") == 0);

  size_t ws = 0, saved = 0;
  CHECK(hstu_workspace_size(&c, 4, 1000, &ws, &saved) == HSTU_OK);
  CHECK(ws > 0 && saved > 0);
  size_t off[HSTU_SAVED_COUNT + 1];
  CHECK(hstu_saved_layout(&c, 1000, off) == HSTU_OK);
  CHECK(off[HSTU_SAVED_COUNT] == saved);
  /* Pre and G: T x 4d bf16 each */
  CHECK(off[HSTU_SAVED_G] - off[HSTU_SAVED_PRE] >= (size_t)1000 * 4 * 256 * 2);

  /* bf16 heads of 32: the attention workspace adds the zero-padded V|Q|K */
  hstu_config c32 = c, c64 = c;
  c32.d_model = 64;  c32.head_dim = 32;
  c64.d_model = 128; c64.head_dim = 64;
  const size_t sched = hstu_attention_workspace_size(&c64, 4, 1000);
  CHECK(hstu_attention_workspace_size(&c32, 4, 1000) ==
        (sched + 255) / 256 * 256 + (size_t)1000 * 3 * 2 * 64 * 2);

  /* host-checkable errors return before any launch */
  hstu_weights w;
  memset(&w, 0, sizeof(w));
  int64_t offs[5] = {0, 0, 0, 0, 0};
  CHECK(hstu_fwd(&c, &w, NULL, offs, 4, 10, NULL, NULL, NULL, NULL, NULL, NULL, 0, 0) ==
        HSTU_ERR_INVALID);
  CHECK(hstu_fwd(NULL, &w, NULL, offs, 4, 10, NULL, NULL, NULL, NULL, NULL, NULL, 0, 0) ==
        HSTU_ERR_INVALID);
  c.head_dim = 48; c.d_model = 96;
  CHECK(hstu_workspace_size(&c, 4, 10, &ws, &saved) == HSTU_ERR_UNSUPPORTED);
  printf("c host ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_links_and_runs_host_entry_points():
    lib = build.build()
    libdir = os.path.dirname(lib)
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "host.c")
        exe = os.path.join(tmp, "host")
        with open(src, "w") as f:
            f.write(PROGRAM)
        cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
               "-I", os.path.join(CUDA, "include"), src, "-o", exe, "-L", libdir, "-lhstu",
               "-Wl,-rpath," + libdir, "-L", os.path.join(CUDA, "lib64"), "-lcudart",
               "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "c host ok" in r.stdout

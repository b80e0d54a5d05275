"""The header as a C program sees it, without a GPU: include/da.h compiles as strict C99 with
every warning an error, and a C program linked against libda.so gets the same descriptor,
workspace sizes, argument checks and status strings the binding gets.  Only calls that return
before any CUDA call are made."""

import os
import subprocess

import pytest

from conftest import ROOT

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "da.h"

static int fails = 0;
#define CHECK(c) do { if (!(c)) { printf("FAIL line %d: %s\n", __LINE__, #c); ++fails; } } while (0)

int main(void) {
  da_problem p;
  da_plan_desc d, s;
  size_t ws = 0, po = 0, pl = 0;
  int64_t off[7];
  memset(&p, 0, sizeof p);
  p.batch = 32; p.num_q_heads = 64; p.num_kv_heads = 8; p.head_dim = 128; p.page_size = 64;
  p.max_pages_per_req = 250; p.num_pages = 8400; p.scale = 0.08838834764831845f; p.q_len = 1;

  CHECK(da_plan_desc_init(&p, DA_PLAN_DYNAMIC, 64, 37, &d) == DA_OK);
  CHECK(d.kind == DA_PLAN_DYNAMIC && d.batch == 32 && d.tile_tokens == 64 && d.num_ctas == 37);
  CHECK(d.splits == 0 && d.max_segments == 37 + 32 - 1 && d.num_kv_heads == 8 && d.merge_in_decode == 0);
  CHECK(d.out_format == DA_OUT_BF16 && d.start_cost == 2);
  CHECK(da_plan_workspace_size(&p, 64, 37, &ws, &po, &pl) == DA_OK);
  CHECK(po == (size_t)d.max_segments * 64 * 128 * 4);
  CHECK(da_workspace_size(&p, &d, &ws, &po, &pl) == DA_OK);
  CHECK(po == (size_t)d.max_segments * 64 * 128 * 4 && pl == (size_t)d.max_segments * 64 * 4);
  CHECK(ws % 16 == 0 && ws > 0);
  CHECK(da_workspace_offsets(&d, off) == DA_OK && off[0] == 0 && (size_t)off[6] * 4 == ws);
  CHECK(da_workspace_size(&p, &d, NULL, NULL, NULL) == DA_OK);

  CHECK(da_plan_desc_init(&p, DA_PLAN_STATIC, 32, 3, &s) == DA_OK);
  CHECK(s.kind == DA_PLAN_STATIC && s.num_ctas == 96 && s.splits == 3 && s.max_segments == 96);
  CHECK(s.start_cost == 0);
  s.start_cost = 1;  /* start units belong to dynamic plans */
  CHECK(da_workspace_size(&p, &s, &ws, &po, &pl) == DA_ERR_INVALID_ARG);
  s.start_cost = 0;
  d.start_cost = -1;
  CHECK(da_workspace_size(&p, &d, &ws, &po, &pl) == DA_ERR_INVALID_ARG);
  d.start_cost = 0;  /* the tiles-only plan: same sizes */
  CHECK(da_workspace_size(&p, &d, &ws, &po, &pl) == DA_OK);
  d.start_cost = 2;

  /* fp32 output: every request goes through the combine, which cannot run inside the decode */
  d.out_format = DA_OUT_F32;
  CHECK(da_workspace_size(&p, &d, &ws, &po, &pl) == DA_OK);
  d.merge_in_decode = 1;
  CHECK(da_workspace_size(&p, &d, &ws, &po, &pl) == DA_ERR_INVALID_ARG);
  d.merge_in_decode = 0; d.out_format = 2;
  CHECK(da_workspace_size(&p, &d, &ws, &po, &pl) == DA_ERR_INVALID_ARG);
  d.out_format = DA_OUT_BF16;

  /* argument checks: nothing is enqueued */
  CHECK(da_plan(&p, &s, (const int32_t*)16, (void*)256, 1 << 20, NULL) == DA_ERR_INVALID_ARG);
  CHECK(da_plan(&p, &d, (const int32_t*)16, (void*)256, 64, NULL) == DA_ERR_WORKSPACE);
  CHECK(da_plan(&p, &d, NULL, (void*)256, 1 << 20, NULL) == DA_ERR_INVALID_ARG);
  CHECK(da_read_status(NULL, NULL, NULL, NULL) == DA_ERR_INVALID_ARG);
  p.num_q_heads = 60;
  CHECK(da_plan_desc_init(&p, DA_PLAN_DYNAMIC, 64, 37, &d) == DA_ERR_INVALID_ARG);
  p.num_q_heads = 64; p.head_dim = 96;
  CHECK(da_plan_desc_init(&p, DA_PLAN_DYNAMIC, 64, 37, &d) == DA_ERR_UNSUPPORTED);

  /* balance tables: sizes, and a table from block times (host only) */
  p.head_dim = 128;
  CHECK(da_plan_desc_init(&p, DA_PLAN_DYNAMIC, 64, 37, &d) == DA_OK);
  CHECK(d.balance == NULL && d.block_times == NULL);
  {
    size_t words = 0;
    int64_t times[8 * 37 * 2];
    int32_t w[37], perm[8 * 37];
    CHECK(da_balance_words(&d, &words) == DA_OK && words == 4 + 37 + 8 * 37);
    CHECK(da_balance_words(&s, &words) == DA_ERR_INVALID_ARG);
    for (int i = 0; i < 8 * 37; ++i) {
      times[2 * i] = 1000;
      times[2 * i + 1] = 1000 + 100000 + (i % 37) * 100;  /* block x of every row: slower as x grows */
    }
    CHECK(da_balance_from_times(&d, times, NULL, NULL, w, perm) == DA_OK);
    CHECK(perm[0] == 36 && perm[36] == 0 && w[0] < w[36]);  /* the slowest block runs CTA 0 */
    perm[1] = perm[0];  /* not a permutation: refused before any copy */
    CHECK(da_balance_set(&d, w, perm, (int32_t*)256, NULL) == DA_ERR_INVALID_ARG);
  }
  CHECK(strlen(da_status_string(DA_OK)) > 0 && strlen(da_status_string(DA_ERR_WORKSPACE)) > 0);
  CHECK(strlen(da_dev_status_string(DA_DEV_TIMEOUT)) > 0 && strlen(da_dev_status_string(DA_DEV_BAD_BALANCE)) > 0);
  printf("%s\n", fails ? "C ABI FAILED" : "C ABI OK");
  return fails != 0;
}
"""


def test_header_compiles_as_c99_and_links(da_lib, tmp_path):
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(da_lib.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(da_lib.LIB_PATH),
           "-Wl,-rpath," + libdir]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        pytest.fail(f"C build failed:\n{res.stderr}")
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "C ABI OK" in run.stdout

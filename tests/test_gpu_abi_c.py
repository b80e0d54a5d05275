"""One decode step run by a C program through the C ABI, on the GPU.

The program is plain C99 linked against libda.so and the CUDA runtime.  It reads
the tiny batch (written here from the seeded generator), puts the caches on the
device, and runs da_decode_step_host twice from host buffers: once from ordinary
malloc'd memory (the call copies inputs in and outputs back on the stream) and once
from cudaMallocHost memory (the plan launch reads the inputs over the bus and the
kernels write out/lse in place).  It writes both results; this test compares them
with the fp64 oracle and with each other, bit for bit.
"""

import os
import subprocess

import numpy as np
import pytest
import torch

from conftest import ROOT
from gpu_helpers import LSE_ATOL, OUT_ATOL, OUT_RTOL
from variable_length_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu

PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime_api.h>
#include "da.h"

static void* slurp(const char* dir, const char* name, size_t bytes) {
  char path[1024];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  if (!f) { fprintf(stderr, "cannot open %s\n", path); exit(2); }
  void* p = malloc(bytes ? bytes : 1);
  if (fread(p, 1, bytes, f) != bytes) { fprintf(stderr, "short read %s\n", path); exit(2); }
  fclose(f);
  return p;
}

static void spill(const char* dir, const char* name, const void* p, size_t bytes) {
  char path[1024];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(p, 1, bytes, f) != bytes) { fprintf(stderr, "cannot write %s\n", path); exit(2); }
  fclose(f);
}

#define CU(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
  fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_)); return 3; } } while (0)
#define DA(x) do { int r_ = (x); if (r_ != DA_OK) { \
  fprintf(stderr, "%s: %s (cuda %d)\n", #x, da_status_string(r_), (int)da_last_cuda_error()); return 4; } } while (0)

int main(int argc, char** argv) {
  if (argc != 2) return 1;
  const char* dir = argv[1];
  int32_t* hdr = (int32_t*)slurp(dir, "problem.bin", 8 * sizeof(int32_t));
  da_problem p;
  memset(&p, 0, sizeof p);
  p.batch = hdr[0]; p.num_q_heads = hdr[1]; p.num_kv_heads = hdr[2]; p.head_dim = hdr[3];
  p.page_size = hdr[4]; p.max_pages_per_req = hdr[5]; p.num_pages = hdr[6]; p.q_len = 1;
  float* scale = (float*)slurp(dir, "scale.bin", sizeof(float));
  p.scale = *scale;
  const int32_t width = hdr[7];
  const size_t B = (size_t)p.batch, rows = B * (size_t)p.num_q_heads;
  const size_t q_bytes = rows * (size_t)p.head_dim * 2, bt_bytes = B * (size_t)p.max_pages_per_req * 4;
  const size_t kv_bytes = (size_t)p.num_pages * p.num_kv_heads * p.page_size * p.head_dim * 2;
  void* q = slurp(dir, "q.bin", q_bytes);
  void* k = slurp(dir, "k.bin", kv_bytes);
  void* v = slurp(dir, "v.bin", kv_bytes);
  int32_t* bt = (int32_t*)slurp(dir, "block_table.bin", bt_bytes);
  int32_t* sl = (int32_t*)slurp(dir, "seq_lens.bin", B * 4);

  da_plan_desc d;
  size_t ws_b = 0, po_b = 0, pl_b = 0;
  DA(da_plan_desc_init(&p, DA_PLAN_DYNAMIC, 16, width, &d));
  DA(da_workspace_size(&p, &d, &ws_b, &po_b, &pl_b));
  void *k_d, *v_d, *q_d, *out_d, *ws, *pinned;
  int32_t *bt_d, *sl_d;
  float *po, *pl, *lse_d;
  CU(cudaMalloc(&k_d, kv_bytes));
  CU(cudaMalloc(&v_d, kv_bytes));
  CU(cudaMalloc(&q_d, q_bytes));
  CU(cudaMalloc((void**)&bt_d, bt_bytes));
  CU(cudaMalloc((void**)&sl_d, B * 4));
  CU(cudaMalloc(&ws, ws_b));
  CU(cudaMalloc((void**)&po, po_b));
  CU(cudaMalloc((void**)&pl, pl_b));
  CU(cudaMalloc(&out_d, q_bytes));
  CU(cudaMalloc((void**)&lse_d, rows * 4));
  CU(cudaMemcpy(k_d, k, kv_bytes, cudaMemcpyHostToDevice));
  CU(cudaMemcpy(v_d, v, kv_bytes, cudaMemcpyHostToDevice));
  cudaStream_t s;
  CU(cudaStreamCreate(&s));

  /* 1: ordinary host memory -- the call copies in and out on the stream */
  void* out_h = malloc(q_bytes);
  float* lse_h = (float*)malloc(rows * 4);
  memset(out_h, 0xFF, q_bytes);
  DA(da_decode_step_host(&p, &d, q, bt, sl, k_d, v_d, NULL, NULL, q_d, bt_d, sl_d, ws, ws_b, po, pl, out_d, lse_d,
                         out_h, lse_h, (void*)s));
  CU(cudaStreamSynchronize(s));
  int32_t st = -1, bad = -2;
  DA(da_read_status(ws, &st, &bad, (void*)s));
  if (st != DA_DEV_OK || bad != -1) { fprintf(stderr, "device status %d / %d\n", st, bad); return 5; }
  spill(dir, "out_copy.bin", out_h, q_bytes);
  spill(dir, "lse_copy.bin", lse_h, rows * 4);

  /* 2: page-locked, mapped host memory -- no copy calls, the kernels read and write it in place */
  const size_t off_q = 0, off_bt = (q_bytes + 255) / 256 * 256, off_sl = off_bt + (bt_bytes + 255) / 256 * 256;
  const size_t off_out = off_sl + (B * 4 + 255) / 256 * 256, off_lse = off_out + (q_bytes + 255) / 256 * 256;
  const size_t total = off_lse + rows * 4;
  CU(cudaMallocHost(&pinned, total));
  unsigned char* base = (unsigned char*)pinned;
  memcpy(base + off_q, q, q_bytes);
  memcpy(base + off_bt, bt, bt_bytes);
  memcpy(base + off_sl, sl, B * 4);
  memset(base + off_out, 0xFF, q_bytes);
  CU(cudaMemset(out_d, 0xFF, q_bytes));
  DA(da_decode_step_host(&p, &d, base + off_q, (int32_t*)(base + off_bt), (int32_t*)(base + off_sl), k_d, v_d,
                         NULL, NULL, q_d, bt_d, sl_d, ws, ws_b, po, pl, out_d, lse_d, base + off_out,
                         (float*)(base + off_lse), (void*)s));
  CU(cudaStreamSynchronize(s));
  DA(da_read_status(ws, &st, &bad, (void*)s));
  if (st != DA_DEV_OK || bad != -1) { fprintf(stderr, "device status %d / %d\n", st, bad); return 5; }
  spill(dir, "out_mapped.bin", base + off_out, q_bytes);
  spill(dir, "lse_mapped.bin", base + off_lse, rows * 4);

  CU(cudaFreeHost(pinned));
  CU(cudaStreamDestroy(s));
  cudaFree(k_d); cudaFree(v_d); cudaFree(q_d); cudaFree(bt_d); cudaFree(sl_d); cudaFree(ws);
  cudaFree(po); cudaFree(pl); cudaFree(out_d); cudaFree(lse_d);
  free(q); free(k); free(v); free(bt); free(sl); free(out_h); free(lse_h); free(hdr); free(scale);
  printf("C STEP OK\n");
  return 0;
}
"""


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_c_program_runs_a_step_from_host_buffers(da_lib, oracle_lib, tmp_path):
    w = W.tiny()
    pr = w.problem
    width = 3
    np.array([pr.batch, pr.num_q_heads, pr.num_kv_heads, pr.head_dim, pr.page_size, pr.max_pages_per_req,
              pr.num_pages, width], np.int32).tofile(tmp_path / "problem.bin")
    np.array([pr.scale], np.float32).tofile(tmp_path / "scale.bin")
    _bits(w.q).tofile(tmp_path / "q.bin")
    _bits(w.k_cache).tofile(tmp_path / "k.bin")
    _bits(w.v_cache).tofile(tmp_path / "v.bin")
    np.ascontiguousarray(w.block_table, np.int32).tofile(tmp_path / "block_table.bin")
    np.ascontiguousarray(w.seq_lens, np.int32).tofile(tmp_path / "seq_lens.bin")

    src = tmp_path / "step.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "step"
    libdir = os.path.dirname(da_lib.LIB_PATH)
    cuda = "/usr/local/cuda"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-I",
           f"{cuda}/include", str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(da_lib.LIB_PATH),
           f"-Wl,-rpath,{libdir}", "-L", f"{cuda}/lib64", "-lcudart", f"-Wl,-rpath,{cuda}/lib64"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        pytest.fail(f"C build failed:\n{res.stderr}")
    run = subprocess.run([str(exe), str(tmp_path)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "C STEP OK" in run.stdout, run.stdout + run.stderr

    B, Hq, d = pr.batch, pr.num_q_heads, pr.head_dim
    ref, ref_lse, st = oracle_lib.attention(w.q, w.k_cache, w.v_cache, w.block_table, w.seq_lens, scale=pr.scale)
    assert st == oracle_lib.OK
    outs = {}
    for kind in ("copy", "mapped"):
        raw = np.fromfile(tmp_path / f"out_{kind}.bin", np.uint16).reshape(B, Hq, d)
        out = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).double().numpy()
        lse = np.fromfile(tmp_path / f"lse_{kind}.bin", np.float32).reshape(B, Hq).astype(np.float64)
        outs[kind] = (raw, lse)
        assert np.all(np.isfinite(out))
        assert np.all(np.abs(out - ref) <= OUT_ATOL + OUT_RTOL * np.abs(ref)), kind
        assert np.all(np.abs(lse - ref_lse) <= LSE_ATOL), kind
    # both ways of moving the inputs and outputs run the same plan and kernels: same bits
    assert np.array_equal(outs["copy"][0], outs["mapped"][0])
    assert np.array_equal(outs["copy"][1], outs["mapped"][1])

// append_rows.cuh -- the per-request body of the KV append, shared by the append
// kernel and the fused plan + append kernel.
#pragma once

#include "da_internal.cuh"

namespace da {

// Write request b's newest K/V rows into its page: seq_lens[b] already counts the
// new token, so the rows go to position seq_lens[b] - 1.  Threads [0, nthreads) of
// the block move 16-byte pieces of the rows of all KV heads.  A bad length or page
// id is recorded in the optional status pair and the row skipped.
__device__ __forceinline__ void append_request_rows(const AppendParams& p, int b, int tid, int nthreads) {
  const int L = p.seq_lens[b];
  if (L == 0) return;
  if (L < 0 || (int64_t)L > p.capacity_tokens) {
    if (tid == 0 && p.status && atomicCAS(&p.status[0], DA_DEV_OK, DA_DEV_BAD_SEQLEN) == DA_DEV_OK)
      atomicExch(&p.status[1], b);
    return;
  }
  const int pos = L - 1;
  const int page = p.block_table[(int64_t)b * p.max_pages_per_req + pos / p.page_size];
  if (page < 0 || page >= p.num_pages) {
    if (tid == 0 && p.status && atomicCAS(&p.status[0], DA_DEV_OK, DA_DEV_BAD_PAGE) == DA_DEV_OK)
      atomicExch(&p.status[1], b);
    return;
  }
  const int slot = pos % p.page_size;
  const int per_row = p.head_dim / 8;  // 16-byte pieces per row
  const int pieces = p.num_kv_heads * per_row;
  for (int i = tid; i < pieces; i += nthreads) {
    const int g = i / per_row, c = i - g * per_row;
    const int64_t src = ((int64_t)b * p.num_kv_heads + g) * p.head_dim + c * 8;
    const int64_t dst = (((int64_t)page * p.num_kv_heads + g) * p.page_size + slot) * p.head_dim + c * 8;
    reinterpret_cast<uint4*>(p.k_cache)[dst / 8] = __ldg(reinterpret_cast<const uint4*>(p.new_k) + src / 8);
    reinterpret_cast<uint4*>(p.v_cache)[dst / 8] = __ldg(reinterpret_cast<const uint4*>(p.new_v) + src / 8);
  }
}

// Host launcher of the fused plan + append kernel (plan.cu): one grid, block 0 plans,
// the others append.
cudaError_t launch_plan_append(const PlanParams& p, const AppendParams& a, cudaStream_t stream);

}  // namespace da

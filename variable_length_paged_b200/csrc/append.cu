// append.cu -- write each request's newest K/V row into its page.
//
// The step just before decode attention: "Tencent HPC lands in SGLang,
// challenging default inference kernels", section "Why Tencent HPC matters for
// online model serving", notes that request lengths change during decoding
// and the tile mapping is rebuilt each step; every decode step adds one token
// to every live request, and its key and value rows must land in the paged
// cache before attention reads them.
//
// One CTA per request; each thread moves 16-byte pieces of the K and V rows
// of all KV heads.  seq_lens already counts the new token, so request b's row
// goes to position seq_lens[b] - 1.  Bad lengths or page ids are recorded in
// the optional status pair and the row is skipped.
#include "da_internal.cuh"

namespace da {
namespace {

__global__ void __launch_bounds__(128) append_kv_kernel(const AppendParams p) {
  grid_dependency_wait();  // lengths and block table may be written by the previous kernel
  const int b = blockIdx.x;
  const int L = p.seq_lens[b];
  if (L == 0) return;
  if (L < 0 || (int64_t)L > p.capacity_tokens) {
    if (threadIdx.x == 0 && p.status && atomicCAS(&p.status[0], DA_DEV_OK, DA_DEV_BAD_SEQLEN) == DA_DEV_OK)
      atomicExch(&p.status[1], b);
    return;
  }
  const int pos = L - 1;
  const int page = p.block_table[(int64_t)b * p.max_pages_per_req + pos / p.page_size];
  if (page < 0 || page >= p.num_pages) {
    if (threadIdx.x == 0 && p.status && atomicCAS(&p.status[0], DA_DEV_OK, DA_DEV_BAD_PAGE) == DA_DEV_OK)
      atomicExch(&p.status[1], b);
    return;
  }
  const int slot = pos % p.page_size;
  const int per_row = p.head_dim / 8;  // 16-byte pieces per row
  const int pieces = p.num_kv_heads * per_row;
  for (int i = threadIdx.x; i < pieces; i += blockDim.x) {
    const int g = i / per_row, c = i - g * per_row;
    const int64_t src = ((int64_t)b * p.num_kv_heads + g) * p.head_dim + c * 8;
    const int64_t dst = (((int64_t)page * p.num_kv_heads + g) * p.page_size + slot) * p.head_dim + c * 8;
    reinterpret_cast<uint4*>(p.k_cache)[dst / 8] = __ldg(reinterpret_cast<const uint4*>(p.new_k) + src / 8);
    reinterpret_cast<uint4*>(p.v_cache)[dst / 8] = __ldg(reinterpret_cast<const uint4*>(p.new_v) + src / 8);
  }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  if (p.batch == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.batch, 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, append_kv_kernel, p);
}

}  // namespace da

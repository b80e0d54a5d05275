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
#include "append_rows.cuh"
#include "da_internal.cuh"

namespace da {
namespace {

__global__ void __launch_bounds__(128) append_kv_kernel(const AppendParams p) {
  grid_dependency_wait();  // lengths and block table may be written by the previous kernel
  append_request_rows(p, blockIdx.x, threadIdx.x, blockDim.x);
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

// noalloc.cu -- one decode step that allocates nothing.
//
// Some callers cannot allocate device memory where they run a decode step:
// an attention op inside a host framework whose per-call hook must not
// allocate, an engine that has handed nearly all device memory to its
// KV-cache pool up front and has none left to give, or a latency-critical
// path on which a cudaMalloc (which may synchronise the device) is not
// acceptable.  Such callers still own their inputs and outputs, but cannot
// provide the workspace and split partials that da_plan / da_decode_attention
// / da_combine ask for.
//
// This file keeps that scratch in a fixed-size file-scope device array.  The
// array is reserved on every GPU that loads the library's device code and is
// held until the process exits.  Host code cannot use the array's name as a
// device address (on the host it names a stand-in object), so the address is
// looked up once per device with cudaGetSymbolAddress and passed to the
// kernels.
#include <mutex>

#include "da_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_step_scratch[DA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

size_t round_up_256(size_t n) { return (n + 255) / 256 * 256; }

// Device address of g_step_scratch on the current device (looked up on first use).
cudaError_t scratch_address(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_step_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" DA_API int da_decode_step_noalloc(const da_problem* prob, int32_t tile_tokens, int32_t num_ctas,
                                             const void* q, const void* k_cache, const void* v_cache,
                                             const int32_t* block_table, const int32_t* seq_lens, void* out,
                                             float* lse, void* stream) {
  da_plan_desc desc;
  int rc = da_plan_desc_init(prob, DA_PLAN_DYNAMIC, tile_tokens, num_ctas, &desc);
  if (rc != DA_OK) return rc;
  size_t ws_bytes = 0, po_bytes = 0, pl_bytes = 0;
  rc = da_workspace_size(prob, &desc, &ws_bytes, &po_bytes, &pl_bytes);
  if (rc != DA_OK) return rc;
  const size_t ws_r = round_up_256(ws_bytes), po_r = round_up_256(po_bytes), pl_r = round_up_256(pl_bytes);
  if (ws_r + po_r + pl_r > (size_t)DA_NOALLOC_SCRATCH_BYTES) return DA_ERR_WORKSPACE;
  if (prob->batch > 0 && (!q || !k_cache || !v_cache || !block_table || !seq_lens || !out || !lse))
    return DA_ERR_INVALID_ARG;
  // the decode call's alignment rules, checked here so that an error enqueues nothing (not even the plan)
  if (prob->batch > 0 &&
      (reinterpret_cast<uintptr_t>(k_cache) % 16 != 0 || reinterpret_cast<uintptr_t>(v_cache) % 16 != 0 ||
       reinterpret_cast<uintptr_t>(q) % 4 != 0 || reinterpret_cast<uintptr_t>(out) % 8 != 0))
    return DA_ERR_INVALID_ARG;
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) {
    da::set_last_cuda_error(e);
    return DA_ERR_CUDA;
  }
  unsigned char* s = static_cast<unsigned char*>(base);
  void* ws = s;
  float* partial_o = reinterpret_cast<float*>(s + ws_r);
  float* partial_lse = reinterpret_cast<float*>(s + ws_r + po_r);
  // The plan kernel rewrites every scratch word that decode and combine read
  // (header, status, segment list, prefixes), and decode writes every partial
  // that combine reads, so nothing left by an earlier call needs clearing.
  rc = da_plan(prob, &desc, seq_lens, ws, ws_r, stream);
  if (rc != DA_OK) return rc;
  rc = da_decode_attention(prob, &desc, q, k_cache, v_cache, block_table, seq_lens, ws, partial_o, partial_lse, out,
                           lse, stream);
  if (rc != DA_OK) return rc;
  return da_combine(prob, &desc, ws, partial_o, partial_lse, out, lse, stream);
}

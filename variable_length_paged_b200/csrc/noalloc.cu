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
#include <cudaTypedefs.h>

#include <mutex>

#include "prepared_step.cuh"

namespace {

static __device__ __align__(256) unsigned char g_step_scratch[DA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;

// The array's address as resolved on one device, and the id of the context it was resolved
// in.  Context ids are never reused within a process, so a context made after a device reset
// (whose copy of the array may sit elsewhere) never matches an old entry.
struct ScratchEntry {
  void* addr;
  unsigned long long ctx_id;
  bool have_id;
};
ScratchEntry g_scratch[kMaxDevices] = {};

// Driver entry points for the current context's id, looked up once through the runtime.
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};
const CtxFns& ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return f;
}

// Id of the calling thread's current context; false when there is none or it cannot be read.
bool current_ctx_id(unsigned long long* id) {
  const CtxFns& f = ctx_fns();
  CUcontext ctx = nullptr;
  if (!f.get_current || !f.get_id || f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return f.get_id(ctx, id) == CUDA_SUCCESS;
}

size_t round_up_256(size_t n) { return (n + 255) / 256 * 256; }

// Device address of g_step_scratch on the current device.  Looked up with cudaGetSymbolAddress
// (which loads the module into the device's context if needed) the first time on each device,
// and again whenever the device's context is not the one of the last lookup.
cudaError_t scratch_address(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchEntry& ent = g_scratch[dev];
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  if (ent.addr && ent.have_id && have_id && ent.ctx_id == id) {
    *addr = ent.addr;
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_step_scratch);
  if (e != cudaSuccess) return e;
  ent.addr = p;
  ent.have_id = current_ctx_id(&ent.ctx_id);  // the lookup made the primary context current if it was not
  *addr = p;
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
  // the decode call's alignment rules, checked before the first CUDA call (the scratch lookup)
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
  // Every check of the three launches (alignment, tensor maps) runs first, so an
  // error return enqueues nothing unless the CUDA runtime refuses a launch.
  da::PreparedStep st;
  rc = da::prepare_dynamic_step(prob, &desc, q, k_cache, v_cache, block_table, seq_lens, ws, ws_r, partial_o,
                                partial_lse, out, lse, &st);
  if (rc != DA_OK) return rc;
  return da::launch_prepared_step(st, stream);
}

extern "C" DA_API int da_noalloc_read_status(int32_t* dev_status, int32_t* bad_index, void* stream) {
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) {
    da::set_last_cuda_error(e);
    return DA_ERR_CUDA;
  }
  return da_read_status(base, dev_status, bad_index, stream);
}

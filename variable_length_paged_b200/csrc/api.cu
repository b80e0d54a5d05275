// api.cu -- host side of libda.so: argument checks, plan geometry, TMA
// descriptors and launches.  Nothing here allocates, frees or synchronises
// (except da_read_status, documented to synchronise its stream).
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "append_rows.cuh"
#include "da_internal.cuh"
#include "host_inputs.cuh"
#include "prepared_step.cuh"

namespace {

thread_local int32_t g_last_cuda_error = 0;
// failure-path test: limit (ns) for the next decode launch on this thread, which then stalls
thread_local uint64_t g_stall_next_ns = 0;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate pipeline wait

constexpr int kDefaultTile = 64;
constexpr int kCtasPerSm = 2;  // decode kernel residency (shared memory sized for two)
// Start units of a dynamic plan: the fixed cost of starting a request (query load, merge and
// write of its result, about 2 us of one CTA's time on B200) in 64-token tiles of bf16 d 128.
constexpr int32_t kDefaultStartCost = 2;
constexpr int32_t kMaxStartCost = 1 << 16;
constexpr int kMaxRows = 16;  // query heads x queries per request packed on one MMA tile

int q_len_of(const da_problem* p) { return p->q_len > 1 ? p->q_len : 1; }

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int32_t)e;
  return DA_ERR_CUDA;
}

int check_problem(const da_problem* p) {
  if (!p) return DA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->head_dim <= 0 || p->page_size <= 0 ||
      p->max_pages_per_req <= 0 || p->num_pages <= 0)
    return DA_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return DA_ERR_INVALID_ARG;
  if (!(p->scale == p->scale)) return DA_ERR_INVALID_ARG;  // NaN scale
  if (p->head_dim != 64 && p->head_dim != 128) return DA_ERR_UNSUPPORTED;
  if (p->q_len < 0) return DA_ERR_INVALID_ARG;
  if ((int64_t)(p->num_q_heads / p->num_kv_heads) * q_len_of(p) > kMaxRows) return DA_ERR_UNSUPPORTED;
  if (p->page_size % 16 != 0) return DA_ERR_UNSUPPORTED;
  if ((int64_t)p->num_pages * p->num_kv_heads * p->page_size >= (int64_t)INT_MAX) return DA_ERR_UNSUPPORTED;
  if ((int64_t)p->max_pages_per_req * p->page_size >= (int64_t)INT_MAX) return DA_ERR_UNSUPPORTED;
  return DA_OK;
}

int check_desc(const da_problem* p, const da_plan_desc* d) {
  if (!d) return DA_ERR_INVALID_ARG;
  if (d->batch != p->batch || d->tile_tokens <= 0 || d->tile_tokens % 16 != 0 || d->num_ctas <= 0)
    return DA_ERR_INVALID_ARG;
  if (d->num_kv_heads != p->num_kv_heads || (d->merge_in_decode != 0 && d->merge_in_decode != 1))
    return DA_ERR_INVALID_ARG;
  if (d->out_format != DA_OUT_BF16 && d->out_format != DA_OUT_F32) return DA_ERR_INVALID_ARG;
  if (d->out_format == DA_OUT_F32 && d->merge_in_decode) return DA_ERR_INVALID_ARG;  // the combine writes fp32 out
  if (d->start_cost < 0 || d->start_cost > kMaxStartCost) return DA_ERR_INVALID_ARG;
  if (d->start_cost != 0 && d->kind != DA_PLAN_DYNAMIC) return DA_ERR_INVALID_ARG;
  if (d->balance) {  // a balance table: dynamic plans, 4-byte aligned, within the planner's limit
    if (d->kind != DA_PLAN_DYNAMIC || reinterpret_cast<uintptr_t>(d->balance) % 4 != 0) return DA_ERR_INVALID_ARG;
    if (d->num_ctas > da::kBalanceMaxCtas) return DA_ERR_UNSUPPORTED;
  }
  if (reinterpret_cast<uintptr_t>(d->block_times) % 8 != 0) return DA_ERR_INVALID_ARG;
  if (d->kind == DA_PLAN_DYNAMIC) {
    if (d->splits != 0 || (int64_t)d->max_segments != (int64_t)d->num_ctas + (p->batch > 0 ? p->batch : 1) - 1)
      return DA_ERR_INVALID_ARG;
  } else if (d->kind == DA_PLAN_STATIC) {
    if (d->splits <= 0 || (int64_t)d->num_ctas != (int64_t)p->batch * d->splits || d->max_segments != d->num_ctas)
      return DA_ERR_INVALID_ARG;
  } else {
    return DA_ERR_INVALID_ARG;
  }
  // every tile index and unit count (start units included) stays inside int32
  const int64_t cap = (int64_t)p->max_pages_per_req * p->page_size;
  const int64_t units = (int64_t)p->batch * ((cap + d->tile_tokens - 1) / d->tile_tokens + d->start_cost);
  if (units >= (int64_t)INT_MAX) return DA_ERR_UNSUPPORTED;
  if ((int64_t)d->num_ctas * (units + 1) >= ((int64_t)1 << 62)) return DA_ERR_UNSUPPORTED;
  return DA_OK;
}

size_t ws_words(const da_plan_desc* d) {
  return (size_t)da::ws_layout(d->batch, d->num_ctas, d->max_segments, d->num_kv_heads).total;
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link-time libcuda dependency).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D view of a cache: x = head_dim (inner), y = (page, kv head, slot) rows.
// Box = 128 bytes of columns (the 128-byte swizzle span) x box_rows rows;
// elements are bf16 (2 bytes) or FP8 codes (1 byte).
bool make_cache_map(CUtensorMap* map, const void* base, const da_problem* p, int box_rows, int elem_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)p->head_dim,
                        (cuuint64_t)p->num_pages * (cuuint64_t)p->num_kv_heads * (cuuint64_t)p->page_size};
  cuuint64_t strides[1] = {(cuuint64_t)p->head_dim * (cuuint64_t)elem_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

namespace da {
void set_last_cuda_error(cudaError_t e) { g_last_cuda_error = (int32_t)e; }
}  // namespace da

extern "C" {

DA_API int32_t da_last_cuda_error(void) { return g_last_cuda_error; }

DA_API int da_test_stall_next_decode(uint32_t wait_limit_us) {
  if (wait_limit_us == 0 || wait_limit_us > 2000000u) return DA_ERR_INVALID_ARG;
  g_stall_next_ns = (uint64_t)wait_limit_us * 1000u;
  return DA_OK;
}

DA_API int da_device_num_sms(int32_t* num_sms) {
  if (!num_sms) return DA_ERR_INVALID_ARG;
  int dev = 0, n = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  *num_sms = n;
  return DA_OK;
}

DA_API int da_plan_desc_init(const da_problem* prob, int32_t kind, int32_t tile_tokens, int32_t width,
                             da_plan_desc* desc) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  if (!desc || width < 0 || tile_tokens < 0) return DA_ERR_INVALID_ARG;
  if (kind != DA_PLAN_DYNAMIC && kind != DA_PLAN_STATIC) return DA_ERR_INVALID_ARG;
  const int T = tile_tokens == 0 ? kDefaultTile : tile_tokens;
  if (T % 16 != 0) return DA_ERR_UNSUPPORTED;
  int w = width;
  if (w == 0) {
    int32_t sms = 0;
    rc = da_device_num_sms(&sms);
    if (rc != DA_OK) return rc;
    const int slots = sms * kCtasPerSm;
    if (kind == DA_PLAN_DYNAMIC) {
      w = slots / prob->num_kv_heads;
      if (w < 1) w = 1;
    } else {
      const int64_t per = (int64_t)(prob->batch > 0 ? prob->batch : 1) * prob->num_kv_heads;
      int64_t s = (slots + per - 1) / per;
      w = (int)(s < 1 ? 1 : s > 64 ? 64 : s);
    }
  }
  da_plan_desc d;
  d.kind = kind;
  d.batch = prob->batch;
  d.tile_tokens = T;
  d.num_kv_heads = prob->num_kv_heads;
  d.merge_in_decode = 0;
  d.out_format = DA_OUT_BF16;
  d.start_cost = kind == DA_PLAN_DYNAMIC ? kDefaultStartCost : 0;
  d.balance = nullptr;
  d.block_times = nullptr;
  if (kind == DA_PLAN_DYNAMIC) {
    d.num_ctas = w;
    d.splits = 0;
    const int64_t ms = (int64_t)w + (prob->batch > 0 ? prob->batch : 1) - 1;
    if (ms >= INT_MAX) return DA_ERR_UNSUPPORTED;
    d.max_segments = (int32_t)ms;
  } else {
    const int64_t n = (int64_t)prob->batch * w;
    if (n >= INT_MAX / 4) return DA_ERR_UNSUPPORTED;
    if (n == 0) return DA_ERR_INVALID_ARG;  // a static grid needs at least one request
    d.num_ctas = (int32_t)n;
    d.splits = w;
    d.max_segments = (int32_t)n;
  }
  rc = check_desc(prob, &d);
  if (rc != DA_OK) return rc;
  *desc = d;
  return DA_OK;
}

DA_API int da_workspace_size(const da_problem* prob, const da_plan_desc* desc, size_t* ws_bytes,
                             size_t* partial_o_bytes, size_t* partial_lse_bytes) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  rc = check_desc(prob, desc);
  if (rc != DA_OK) return rc;
  if (ws_bytes) *ws_bytes = ws_words(desc) * 4;
  const size_t rows = (size_t)q_len_of(prob) * prob->num_q_heads;
  if (partial_o_bytes) *partial_o_bytes = (size_t)desc->max_segments * rows * prob->head_dim * 4;
  if (partial_lse_bytes) *partial_lse_bytes = (size_t)desc->max_segments * rows * 4;
  return DA_OK;
}

DA_API int da_plan_workspace_size(const da_problem* prob, int32_t tile_tokens, int32_t num_ctas, size_t* ws_bytes,
                                  size_t* partial_o_bytes, size_t* partial_lse_bytes) {
  da_plan_desc d;
  const int rc = da_plan_desc_init(prob, DA_PLAN_DYNAMIC, tile_tokens, num_ctas, &d);
  return rc != DA_OK ? rc : da_workspace_size(prob, &d, ws_bytes, partial_o_bytes, partial_lse_bytes);
}

DA_API int da_workspace_offsets(const da_plan_desc* desc, int64_t off[7]) {
  if (!desc || !off || desc->batch < 0 || desc->num_ctas <= 0 || desc->max_segments <= 0 || desc->num_kv_heads <= 0)
    return DA_ERR_INVALID_ARG;
  const da::WsLayout L = da::ws_layout(desc->batch, desc->num_ctas, desc->max_segments, desc->num_kv_heads);
  off[0] = L.hdr;
  off[1] = L.segs;
  off[2] = L.req_tile_prefix;
  off[3] = L.req_seg_begin;
  off[4] = L.cta_seg_begin;
  off[5] = L.req_done;
  off[6] = L.total;
  return DA_OK;
}

// Checks a plan call and fills its kernel parameters; enqueues nothing.
static int plan_prepare(const da_problem* prob, const da_plan_desc* desc, const int32_t* seq_lens, void* ws,
                        size_t ws_bytes, int kind, da::PlanParams* p) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  rc = check_desc(prob, desc);
  if (rc != DA_OK) return rc;
  if (desc->kind != kind) return DA_ERR_INVALID_ARG;
  if (!ws || (prob->batch > 0 && !seq_lens)) return DA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % 16 != 0) return DA_ERR_INVALID_ARG;
  if (ws_bytes < ws_words(desc) * 4) return DA_ERR_WORKSPACE;
  p->seq_lens = seq_lens;
  p->ws = static_cast<int32_t*>(ws);
  p->batch = prob->batch;
  p->tile_tokens = desc->tile_tokens;
  p->width = kind == DA_PLAN_DYNAMIC ? desc->num_ctas : desc->splits;
  p->max_segments = desc->max_segments;
  p->num_ctas = desc->num_ctas;
  p->num_kv_heads = prob->num_kv_heads;
  p->capacity_tokens = (int64_t)prob->max_pages_per_req * prob->page_size;
  p->start_cost = kind == DA_PLAN_DYNAMIC ? desc->start_cost : 0;
  p->balance = kind == DA_PLAN_DYNAMIC ? desc->balance : nullptr;
  return DA_OK;
}

static int plan_launch(const da::PlanParams& p, int kind, void* stream) {
  cudaError_t e = kind == DA_PLAN_DYNAMIC ? da::launch_plan_dynamic(p, static_cast<cudaStream_t>(stream))
                                          : da::launch_plan_static(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DA_OK : cuda_fail(e);
}

static int plan_common(const da_problem* prob, const da_plan_desc* desc, const int32_t* seq_lens, void* ws,
                       size_t ws_bytes, void* stream, int kind) {
  da::PlanParams p;
  const int rc = plan_prepare(prob, desc, seq_lens, ws, ws_bytes, kind, &p);
  return rc != DA_OK ? rc : plan_launch(p, kind, stream);
}

DA_API int da_plan(const da_problem* prob, const da_plan_desc* desc, const int32_t* seq_lens, void* ws,
                   size_t ws_bytes, void* stream) {
  return plan_common(prob, desc, seq_lens, ws, ws_bytes, stream, DA_PLAN_DYNAMIC);
}

DA_API int da_static_plan(const da_problem* prob, const da_plan_desc* desc, const int32_t* seq_lens, void* ws,
                          size_t ws_bytes, void* stream) {
  return plan_common(prob, desc, seq_lens, ws, ws_bytes, stream, DA_PLAN_STATIC);
}

// Checks a decode call and fills its kernel parameters and tensor maps; enqueues
// nothing.  Call only with batch > 0.
static int decode_prepare(const da_problem* prob, const da_plan_desc* desc, const void* q, const void* k_cache,
                          const void* v_cache, const float* k_scale, const float* v_scale,
                          const int32_t* block_table, const int32_t* seq_lens, const void* ws, float* partial_o,
                          float* partial_lse, void* out, float* lse, bool fp8, da::DecodeParams* pp,
                          CUtensorMap maps[4]) {
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !ws || !partial_o || !partial_lse || !out || !lse)
    return DA_ERR_INVALID_ARG;
  if (fp8 && (!k_scale || !v_scale)) return DA_ERR_INVALID_ARG;
  const bool out_f32 = desc->out_format == DA_OUT_F32;
  if (reinterpret_cast<uintptr_t>(k_cache) % 16 != 0 || reinterpret_cast<uintptr_t>(v_cache) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(q) % (fp8 ? 8 : 4) != 0 || reinterpret_cast<uintptr_t>(out) % (out_f32 ? 16 : 8) != 0 ||
      reinterpret_cast<uintptr_t>(partial_o) % 16 != 0 || reinterpret_cast<uintptr_t>(ws) % 16 != 0)
    return DA_ERR_INVALID_ARG;
  const int eb = fp8 ? 1 : 2;
  if (!make_cache_map(&maps[0], k_cache, prob, 64, eb) || !make_cache_map(&maps[1], v_cache, prob, 64, eb) ||
      !make_cache_map(&maps[2], k_cache, prob, 16, eb) || !make_cache_map(&maps[3], v_cache, prob, 16, eb))
    return cuda_fail(cudaErrorInvalidValue);
  da::DecodeParams& p = *pp;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.ws = static_cast<const int32_t*>(ws);
  p.partial_o = partial_o;
  p.partial_lse = partial_lse;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.batch = prob->batch;
  p.num_q_heads = prob->num_q_heads;
  p.num_kv_heads = prob->num_kv_heads;
  p.group = prob->num_q_heads / prob->num_kv_heads;
  p.page_size = prob->page_size;
  p.max_pages_per_req = prob->max_pages_per_req;
  p.num_pages = prob->num_pages;
  p.tile_tokens = desc->tile_tokens;
  p.num_ctas = desc->num_ctas;
  p.max_segments = desc->max_segments;
  p.kind = desc->kind;
  p.capacity_tokens = (int64_t)prob->max_pages_per_req * prob->page_size;
  p.scale_log2 = prob->scale * 1.4426950408889634f;
  p.q_len = q_len_of(prob);
  // several queries per request, or more than 8 heads per group, take the kernel that maps
  // (query, head) rows over all 16 MMA rows; plain decode with G <= 8 uses the upper 8
  p.full_rows = (p.q_len > 1 || p.group > 8) ? 1 : 0;
  p.merge_in_decode = desc->merge_in_decode;
  p.out_f32 = out_f32 ? 1 : 0;
  p.stall_producer = g_stall_next_ns != 0 ? 1 : 0;
  p.wait_limit_ns = g_stall_next_ns != 0 ? g_stall_next_ns : kWaitLimitNs;
  g_stall_next_ns = 0;  // one launch only
  // the balance table's placement part; the kernel follows it only if the plan took the table
  p.cta_perm = desc->balance ? desc->balance + da::kBalanceHeader + desc->num_ctas : nullptr;
  p.block_times = desc->block_times;
  return DA_OK;
}

// FP8 plain decode (one query, at most 8 heads per KV head, merge by da_combine) runs
// on the tcgen05 kernel; multi-query and in-decode merge use the warp-MMA kernel.
static int decode_launch(const da::DecodeParams& p, int head_dim, const CUtensorMap maps[4], bool fp8,
                         void* stream) {
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (!fp8)
    e = da::launch_decode(p, head_dim, maps, s);
  else if (head_dim == 128 && p.full_rows == 0 && p.merge_in_decode == 0)
    e = da::launch_decode_fp8_tc(p, maps, s);
  else
    e = da::launch_decode_fp8(p, head_dim, maps, s);
  return e == cudaSuccess ? DA_OK : cuda_fail(e);
}

static int decode_common(const da_problem* prob, const da_plan_desc* desc, const void* q, const void* k_cache,
                         const void* v_cache, const float* k_scale, const float* v_scale,
                         const int32_t* block_table, const int32_t* seq_lens, const void* ws, float* partial_o,
                         float* partial_lse, void* out, float* lse, void* stream, bool fp8) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  rc = check_desc(prob, desc);
  if (rc != DA_OK) return rc;
  if (fp8 && prob->head_dim != 128) return DA_ERR_UNSUPPORTED;
  if (prob->batch == 0) return DA_OK;
  da::DecodeParams p;
  CUtensorMap maps[4];
  rc = decode_prepare(prob, desc, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, ws, partial_o,
                      partial_lse, out, lse, fp8, &p, maps);
  return rc != DA_OK ? rc : decode_launch(p, prob->head_dim, maps, fp8, stream);
}

DA_API int da_decode_attention(const da_problem* prob, const da_plan_desc* desc, const void* q,
                               const void* k_cache, const void* v_cache, const int32_t* block_table,
                               const int32_t* seq_lens, const void* ws, float* partial_o, float* partial_lse,
                               void* out, float* lse, void* stream) {
  return decode_common(prob, desc, q, k_cache, v_cache, nullptr, nullptr, block_table, seq_lens, ws, partial_o,
                       partial_lse, out, lse, stream, false);
}

DA_API int da_decode_attention_fp8(const da_problem* prob, const da_plan_desc* desc, const void* q,
                                   const void* k_cache, const void* v_cache, const float* k_scale,
                                   const float* v_scale, const int32_t* block_table, const int32_t* seq_lens,
                                   const void* ws, float* partial_o, float* partial_lse, void* out, float* lse,
                                   void* stream) {
  return decode_common(prob, desc, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, ws, partial_o,
                       partial_lse, out, lse, stream, true);
}

DA_API int da_decode_step(const da_problem* prob, const da_plan_desc* desc, const void* q, const void* k_cache,
                          const void* v_cache, const float* k_scale, const float* v_scale,
                          const int32_t* block_table, const int32_t* seq_lens, void* ws, size_t ws_bytes,
                          float* partial_o, float* partial_lse, void* out, float* lse, void* stream);

// Checks a combine call and fills its kernel parameters; enqueues nothing.
// Call only with batch > 0.
static int combine_prepare(const da_problem* prob, const da_plan_desc* desc, const void* ws,
                           const float* partial_o, const float* partial_lse, void* out, float* lse,
                           da::CombineParams* p) {
  if (!ws || !partial_o || !partial_lse || !out || !lse) return DA_ERR_INVALID_ARG;
  const bool out_f32 = desc->out_format == DA_OUT_F32;
  if (reinterpret_cast<uintptr_t>(partial_o) % 16 != 0 || reinterpret_cast<uintptr_t>(out) % (out_f32 ? 16 : 8) != 0)
    return DA_ERR_INVALID_ARG;
  p->out_f32 = out_f32 ? 1 : 0;
  p->ws = static_cast<const int32_t*>(ws);
  p->partial_o = partial_o;
  p->partial_lse = partial_lse;
  p->out = static_cast<__nv_bfloat16*>(out);
  p->lse = lse;
  p->batch = prob->batch;
  p->num_q_heads = prob->num_q_heads * q_len_of(prob);  // every (query, head) row merges the same way
  p->num_ctas = desc->num_ctas;
  p->max_segments = desc->max_segments;
  p->num_kv_heads = prob->num_kv_heads;
  return DA_OK;
}

static int combine_launch(const da::CombineParams& p, const da_plan_desc* desc, int head_dim, void* stream) {
  if (desc->merge_in_decode) return DA_OK;  // the decode kernel has finished every request
  cudaError_t e = da::launch_combine(p, head_dim, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DA_OK : cuda_fail(e);
}

DA_API int da_combine(const da_problem* prob, const da_plan_desc* desc, const void* ws, const float* partial_o,
                      const float* partial_lse, void* out, float* lse, void* stream) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  rc = check_desc(prob, desc);
  if (rc != DA_OK) return rc;
  if (prob->batch == 0) return DA_OK;
  da::CombineParams p;
  rc = combine_prepare(prob, desc, ws, partial_o, partial_lse, out, lse, &p);
  return rc != DA_OK ? rc : combine_launch(p, desc, prob->head_dim, stream);
}

DA_API int da_decode_step(const da_problem* prob, const da_plan_desc* desc, const void* q, const void* k_cache,
                          const void* v_cache, const float* k_scale, const float* v_scale,
                          const int32_t* block_table, const int32_t* seq_lens, void* ws, size_t ws_bytes,
                          float* partial_o, float* partial_lse, void* out, float* lse, void* stream) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  rc = check_desc(prob, desc);
  if (rc != DA_OK) return rc;
  if ((k_scale == nullptr) != (v_scale == nullptr)) return DA_ERR_INVALID_ARG;
  const bool fp8 = k_scale != nullptr;
  if (fp8 && prob->head_dim != 128) return DA_ERR_UNSUPPORTED;
  da::PlanParams pp;
  rc = plan_prepare(prob, desc, seq_lens, ws, ws_bytes, desc->kind, &pp);
  if (rc != DA_OK) return rc;
  if (prob->batch == 0) return plan_launch(pp, desc->kind, stream);
  da::DecodeParams dp;
  CUtensorMap maps[4];
  rc = decode_prepare(prob, desc, q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens, ws, partial_o,
                      partial_lse, out, lse, fp8, &dp, maps);
  if (rc != DA_OK) return rc;
  da::CombineParams cp;
  rc = combine_prepare(prob, desc, ws, partial_o, partial_lse, out, lse, &cp);
  if (rc != DA_OK) return rc;
  rc = plan_launch(pp, desc->kind, stream);
  if (rc != DA_OK) return rc;
  rc = decode_launch(dp, prob->head_dim, maps, fp8, stream);
  if (rc != DA_OK) return rc;
  return combine_launch(cp, desc, prob->head_dim, stream);
}

// The device address of host memory that kernels may use in place (page-locked and mapped
// into this device's address space), aligned to `align` bytes; nullptr for any other memory.
static void* mapped_host(const void* ptr, size_t align) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    (void)cudaGetLastError();  // not a pointer the runtime knows: plain host memory
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
  if (reinterpret_cast<uintptr_t>(a.devicePointer) % align != 0) return nullptr;
  return a.devicePointer;
}

DA_API int da_decode_step_host(const da_problem* prob, const da_plan_desc* desc, const void* q_host,
                               const int32_t* block_table_host, const int32_t* seq_lens_host, const void* k_cache,
                               const void* v_cache, const float* k_scale, const float* v_scale, void* q_dev,
                               int32_t* block_table_dev, int32_t* seq_lens_dev, void* ws, size_t ws_bytes,
                               float* partial_o, float* partial_lse, void* out_dev, float* lse_dev, void* out_host,
                               float* lse_host, void* stream) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  rc = check_desc(prob, desc);
  if (rc != DA_OK) return rc;
  if ((k_scale == nullptr) != (v_scale == nullptr)) return DA_ERR_INVALID_ARG;
  const bool fp8 = k_scale != nullptr;
  if (fp8 && prob->head_dim != 128) return DA_ERR_UNSUPPORTED;
  if (prob->batch == 0) return DA_OK;
  if (!q_host || !block_table_host || !seq_lens_host || !out_host || !lse_host) return DA_ERR_INVALID_ARG;
  if (!q_dev || !out_dev || !lse_dev) return DA_ERR_INVALID_ARG;  // required whichever way q, out, lse move
  const size_t B = (size_t)prob->batch;
  const size_t rows = B * (size_t)q_len_of(prob) * (size_t)prob->num_q_heads;
  const size_t q_bytes = rows * (size_t)prob->head_dim * 2;
  const size_t out_bytes = rows * (size_t)prob->head_dim * (desc->out_format == DA_OUT_F32 ? 4 : 2);
  const size_t bt_bytes = B * (size_t)prob->max_pages_per_req * 4;
  // Inputs in mapped page-locked memory need no copy call.  The plan launch brings them in:
  // block 0 reads the lengths and plans, the other blocks copy the block table and a small q
  // (up to kQInLaunch bytes: the bus moves it within the launch).  A larger q is read in place
  // by the decode kernel, which spreads the bus traffic over the K/V stream.  out and lse in
  // mapped memory are written in place by the decode and combine kernels.  Anything else goes
  // through copies on the stream.
  constexpr size_t kQInLaunch = size_t(1) << 20;
  const int32_t* sl_map = static_cast<const int32_t*>(mapped_host(seq_lens_host, 4));
  const void* bt_map = mapped_host(block_table_host, 4);
  const void* q_map = mapped_host(q_host, fp8 ? 8 : 4);
  const bool in_launch = sl_map && bt_map && q_map;
  const bool q_in_place = in_launch && q_bytes > kQInLaunch;
  void* out_map = mapped_host(out_host, 16);
  float* lse_map = static_cast<float*>(mapped_host(lse_host, 16));
  void* out_use = out_map ? out_map : out_dev;
  float* lse_use = lse_map ? lse_map : lse_dev;
  // every check of the three device calls runs before the first copy is enqueued
  da::PlanParams pp;
  rc = plan_prepare(prob, desc, seq_lens_dev, ws, ws_bytes, desc->kind, &pp);
  if (rc != DA_OK) return rc;
  da::DecodeParams dp;
  CUtensorMap maps[4];
  rc = decode_prepare(prob, desc, q_in_place ? q_map : q_dev, k_cache, v_cache, k_scale, v_scale, block_table_dev,
                      seq_lens_dev, ws, partial_o, partial_lse, out_use, lse_use, fp8, &dp, maps);
  if (rc != DA_OK) return rc;
  da::CombineParams cp;
  rc = combine_prepare(prob, desc, ws, partial_o, partial_lse, out_use, lse_use, &cp);
  if (rc != DA_OK) return rc;

  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (in_launch) {
    da::HostInputs hi{};
    hi.seq_lens_host = sl_map;
    hi.seq_lens_dev = seq_lens_dev;
    const void* src[2] = {bt_map, q_map};
    void* dst[2] = {block_table_dev, q_dev};
    const size_t bytes[2] = {bt_bytes, q_bytes};
    for (int k = 0; k < 2; ++k) {
      const bool wide = (reinterpret_cast<uintptr_t>(src[k]) | reinterpret_cast<uintptr_t>(dst[k])) % 16 == 0;
      hi.copies[k].src = src[k];
      hi.copies[k].dst = dst[k];
      hi.copies[k].n16 = wide ? (int64_t)(bytes[k] / 16) : 0;
      hi.copies[k].n4 = (int64_t)((bytes[k] - 16 * (size_t)hi.copies[k].n16) / 4);
    }
    hi.num_copies = q_in_place ? 1 : 2;
    e = da::launch_plan_host(pp, desc->kind, hi, s);
    if (e != cudaSuccess) return cuda_fail(e);
  } else {
    e = cudaMemcpyAsync(seq_lens_dev, seq_lens_host, B * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(block_table_dev, block_table_host, bt_bytes, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(q_dev, q_host, q_bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e);
    rc = plan_launch(pp, desc->kind, stream);
    if (rc != DA_OK) return rc;
  }
  rc = decode_launch(dp, prob->head_dim, maps, fp8, stream);
  if (rc != DA_OK) return rc;
  rc = combine_launch(cp, desc, prob->head_dim, stream);
  if (rc != DA_OK) return rc;
  e = cudaSuccess;
  if (!out_map) e = cudaMemcpyAsync(out_host, out_dev, out_bytes, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && !lse_map) e = cudaMemcpyAsync(lse_host, lse_dev, rows * 4, cudaMemcpyDeviceToHost, s);
  return e == cudaSuccess ? DA_OK : cuda_fail(e);
}

// Checks an append and fills its kernel parameters; enqueues nothing.  Call only with batch > 0.
static int append_prepare(const da_problem* prob, const void* new_k, const void* new_v, const int32_t* block_table,
                          const int32_t* seq_lens, void* k_cache, void* v_cache, int32_t* status,
                          da::AppendParams* p) {
  if (!new_k || !new_v || !block_table || !seq_lens || !k_cache || !v_cache) return DA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(new_k) % 16 != 0 || reinterpret_cast<uintptr_t>(new_v) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(k_cache) % 16 != 0 || reinterpret_cast<uintptr_t>(v_cache) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(status) % 4 != 0)
    return DA_ERR_INVALID_ARG;
  p->new_k = static_cast<const __nv_bfloat16*>(new_k);
  p->new_v = static_cast<const __nv_bfloat16*>(new_v);
  p->block_table = block_table;
  p->seq_lens = seq_lens;
  p->k_cache = static_cast<__nv_bfloat16*>(k_cache);
  p->v_cache = static_cast<__nv_bfloat16*>(v_cache);
  p->status = status;
  p->batch = prob->batch;
  p->num_kv_heads = prob->num_kv_heads;
  p->head_dim = prob->head_dim;
  p->page_size = prob->page_size;
  p->max_pages_per_req = prob->max_pages_per_req;
  p->num_pages = prob->num_pages;
  p->capacity_tokens = (int64_t)prob->max_pages_per_req * prob->page_size;
  return DA_OK;
}

DA_API int da_append_kv(const da_problem* prob, const void* new_k, const void* new_v, const int32_t* block_table,
                        const int32_t* seq_lens, void* k_cache, void* v_cache, int32_t* status, void* stream) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  if (prob->batch == 0) return DA_OK;
  da::AppendParams p;
  rc = append_prepare(prob, new_k, new_v, block_table, seq_lens, k_cache, v_cache, status, &p);
  if (rc != DA_OK) return rc;
  cudaError_t e = da::launch_append(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DA_OK : cuda_fail(e);
}

DA_API int da_plan_append(const da_problem* prob, const da_plan_desc* desc, const int32_t* seq_lens, void* ws,
                          size_t ws_bytes, const void* new_k, const void* new_v, const int32_t* block_table,
                          void* k_cache, void* v_cache, int32_t* status, void* stream) {
  da::PlanParams pp;
  int rc = plan_prepare(prob, desc, seq_lens, ws, ws_bytes, DA_PLAN_DYNAMIC, &pp);
  if (rc != DA_OK) return rc;
  if (prob->batch == 0) return plan_launch(pp, DA_PLAN_DYNAMIC, stream);  // nothing to append
  da::AppendParams ap;
  rc = append_prepare(prob, new_k, new_v, block_table, seq_lens, k_cache, v_cache, status, &ap);
  if (rc != DA_OK) return rc;
  cudaError_t e = da::launch_plan_append(pp, ap, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DA_OK : cuda_fail(e);
}

static int merge_common(int32_t num_parts, int64_t rows, int32_t head_dim, const void* part_out, bool f32,
                        const float* part_lse, void* out, float* lse, void* stream) {
  if (num_parts <= 0 || rows < 0) return DA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return DA_ERR_UNSUPPORTED;
  if (rows == 0) return DA_OK;
  if (!part_out || !part_lse || !out || !lse) return DA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(part_out) % (f32 ? 16 : 8) != 0 || reinterpret_cast<uintptr_t>(out) % 8 != 0)
    return DA_ERR_INVALID_ARG;
  da::MergeParams p;
  p.part_out = f32 ? nullptr : static_cast<const __nv_bfloat16*>(part_out);
  p.part_out_f32 = f32 ? static_cast<const float*>(part_out) : nullptr;
  p.part_lse = part_lse;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.num_parts = num_parts;
  p.rows = rows;
  cudaError_t e = da::launch_merge(p, head_dim, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DA_OK : cuda_fail(e);
}

DA_API int da_merge_partials(int32_t num_parts, int64_t rows, int32_t head_dim, const void* part_out,
                             const float* part_lse, void* out, float* lse, void* stream) {
  return merge_common(num_parts, rows, head_dim, part_out, false, part_lse, out, lse, stream);
}

DA_API int da_merge_partials_f32(int32_t num_parts, int64_t rows, int32_t head_dim, const float* part_out,
                                 const float* part_lse, void* out, float* lse, void* stream) {
  return merge_common(num_parts, rows, head_dim, part_out, true, part_lse, out, lse, stream);
}

DA_API int da_read_status(const void* ws, int32_t* dev_status, int32_t* bad_index, void* stream) {
  if (!ws) return DA_ERR_INVALID_ARG;
  int32_t h[da::kHdrWords];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(h, ws, sizeof h, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev_status) *dev_status = h[da::kHdrStatus];
  if (bad_index) *bad_index = h[da::kHdrBadIndex];
  return DA_OK;
}

// ---- balance tables -------------------------------------------------------------------

static int balance_check_desc(const da_plan_desc* desc) {
  if (!desc || desc->kind != DA_PLAN_DYNAMIC || desc->num_ctas <= 0 || desc->num_kv_heads <= 0)
    return DA_ERR_INVALID_ARG;
  if (desc->num_ctas > da::kBalanceMaxCtas) return DA_ERR_UNSUPPORTED;
  return DA_OK;
}

// weights in range, every row of perm a permutation of 0..C-1
static bool balance_valid(int C, int H, const int32_t* weights, const int32_t* perm) {
  for (int c = 0; c < C; ++c)
    if (weights[c] < 1 || weights[c] > da::kBalanceMaxWeight) return false;
  std::vector<char> seen((size_t)C);
  for (int g = 0; g < H; ++g) {
    std::fill(seen.begin(), seen.end(), 0);
    for (int x = 0; x < C; ++x) {
      const int32_t c = perm[(size_t)g * C + x];
      if (c < 0 || c >= C || seen[(size_t)c]) return false;
      seen[(size_t)c] = 1;
    }
  }
  return true;
}

DA_API int da_balance_words(const da_plan_desc* desc, size_t* words) {
  const int rc = balance_check_desc(desc);
  if (rc != DA_OK) return rc;
  if (!words) return DA_ERR_INVALID_ARG;
  *words = (size_t)da::kBalanceHeader + (size_t)desc->num_ctas * (1 + (size_t)desc->num_kv_heads);
  return DA_OK;
}

DA_API int da_balance_set(const da_plan_desc* desc, const int32_t* weights, const int32_t* perm, int32_t* table,
                          void* stream) {
  const int rc = balance_check_desc(desc);
  if (rc != DA_OK) return rc;
  if (!weights || !perm || !table || reinterpret_cast<uintptr_t>(table) % 4 != 0) return DA_ERR_INVALID_ARG;
  const int C = desc->num_ctas, H = desc->num_kv_heads;
  if (!balance_valid(C, H, weights, perm)) return DA_ERR_INVALID_ARG;
  const int32_t head[da::kBalanceHeader] = {da::kBalanceMagic, C, H, 0};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the header is a stack array (pageable: staged before cudaMemcpyAsync returns); the caller's
  // weights and perm follow the same rule, or, if page-locked, must outlive the copies
  cudaError_t e = cudaMemcpyAsync(table, head, sizeof(head), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(table + da::kBalanceHeader, weights, (size_t)C * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(table + da::kBalanceHeader + C, perm, (size_t)C * H * 4, cudaMemcpyHostToDevice, s);
  return e == cudaSuccess ? DA_OK : cuda_fail(e);
}

DA_API int da_balance_from_times(const da_plan_desc* desc, const int64_t* times, const int32_t* prev_weights,
                                 const int32_t* prev_perm, int32_t* weights, int32_t* perm) {
  const int rc = balance_check_desc(desc);
  if (rc != DA_OK) return rc;
  if (!times || !weights || !perm || (prev_weights == nullptr) != (prev_perm == nullptr)) return DA_ERR_INVALID_ARG;
  const int C = desc->num_ctas, H = desc->num_kv_heads;
  if (prev_weights && !balance_valid(C, H, prev_weights, prev_perm)) return DA_ERR_INVALID_ARG;
  // speed of block (x, g): its CTA's share of the work (the weight it ran with) over its time
  std::vector<double> speed((size_t)C * H);
  for (int g = 0; g < H; ++g) {
    std::vector<double> row;
    for (int x = 0; x < C; ++x) {
      const size_t i = (size_t)g * C + x;
      const int c = prev_perm ? prev_perm[i] : x;
      const double w = prev_weights ? (double)prev_weights[c] : 1.0;
      const int64_t dt = times[2 * i + 1] - times[2 * i];
      speed[i] = dt > 0 ? w / (double)dt : -1.0;
      if (speed[i] > 0) row.push_back(speed[i]);
    }
    double med = 1.0;
    if (!row.empty()) {
      std::nth_element(row.begin(), row.begin() + row.size() / 2, row.end());
      med = row[row.size() / 2];
    }
    for (int x = 0; x < C; ++x)
      if (speed[(size_t)g * C + x] <= 0) speed[(size_t)g * C + x] = med;
  }
  // rank the blocks of each row by speed (ties by index): block x runs CTA rank(x); CTA c's
  // speed is the mean over the rows of the c-th slowest block
  std::vector<double> cta_speed((size_t)C, 0.0);
  std::vector<int> order((size_t)C);
  for (int g = 0; g < H; ++g) {
    const double* sp = speed.data() + (size_t)g * C;
    for (int x = 0; x < C; ++x) order[(size_t)x] = x;
    std::stable_sort(order.begin(), order.end(), [sp](int a, int b) { return sp[a] < sp[b]; });
    for (int r = 0; r < C; ++r) {
      perm[(size_t)g * C + order[(size_t)r]] = r;
      cta_speed[(size_t)r] += sp[order[(size_t)r]] / H;
    }
  }
  double mean = 0.0;
  for (int c = 0; c < C; ++c) mean += cta_speed[(size_t)c] / C;
  for (int c = 0; c < C; ++c) {
    const double w = mean > 0 ? 4096.0 * cta_speed[(size_t)c] / mean : 4096.0;
    weights[c] = (int32_t)std::min<double>(std::max<double>(std::llround(w), 1.0), (double)da::kBalanceMaxWeight);
  }
  return DA_OK;
}

DA_API const char* da_status_string(int32_t code) {
  switch (code) {
    case DA_OK: return "ok";
    case DA_ERR_INVALID_ARG: return "invalid argument";
    case DA_ERR_UNSUPPORTED: return "unsupported problem shape";
    case DA_ERR_CUDA: return "CUDA runtime error";
    case DA_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown return code";
  }
}

DA_API const char* da_dev_status_string(int32_t code) {
  switch (code) {
    case DA_DEV_OK: return "ok";
    case DA_DEV_BAD_SEQLEN: return "sequence length out of range";
    case DA_DEV_BAD_PAGE: return "block-table page id out of range";
    case DA_DEV_TIMEOUT: return "pipeline wait timed out";
    case DA_DEV_BAD_PLAN: return "workspace plan does not match the descriptor";
    case DA_DEV_BAD_BALANCE: return "balance table does not match the descriptor (even split used)";
    default: return "unknown device status";
  }
}

}  // extern "C"

namespace da {

// Every check and parameter block of a dynamic step (plan, bf16 decode, combine) on device
// buffers, before anything is enqueued; launch_prepared_step then only enqueues.
int prepare_dynamic_step(const da_problem* prob, const da_plan_desc* desc, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* block_table, const int32_t* seq_lens, void* ws,
                         size_t ws_bytes, float* partial_o, float* partial_lse, void* out, float* lse,
                         PreparedStep* st) {
  int rc = check_problem(prob);
  if (rc != DA_OK) return rc;
  rc = check_desc(prob, desc);
  if (rc != DA_OK) return rc;
  st->batch = prob->batch;
  st->head_dim = prob->head_dim;
  st->desc = *desc;
  rc = plan_prepare(prob, desc, seq_lens, ws, ws_bytes, DA_PLAN_DYNAMIC, &st->plan);
  if (rc != DA_OK || prob->batch == 0) return rc;
  rc = decode_prepare(prob, desc, q, k_cache, v_cache, nullptr, nullptr, block_table, seq_lens, ws, partial_o,
                      partial_lse, out, lse, false, &st->decode, st->maps);
  if (rc != DA_OK) return rc;
  return combine_prepare(prob, desc, ws, partial_o, partial_lse, out, lse, &st->combine);
}

int launch_prepared_step(const PreparedStep& st, void* stream) {
  int rc = plan_launch(st.plan, DA_PLAN_DYNAMIC, stream);
  if (rc != DA_OK || st.batch == 0) return rc;
  rc = decode_launch(st.decode, st.head_dim, st.maps, false, stream);
  if (rc != DA_OK) return rc;
  return combine_launch(st.combine, &st.desc, st.head_dim, stream);
}

}  // namespace da

// da_internal.cuh -- shared pieces of libda.so: workspace layout, kernel
// parameter blocks, and thin inline-PTX wrappers for the sm_100a features the
// kernels use (mbarrier, TMA tensor loads, ldmatrix, bf16 mma).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "da.h"

namespace da {

// ---- workspace layout (int32 words) ------------------------------------------------------
enum HeaderWord {
  kHdrUnits = 0,
  kHdrSegments = 1,
  kHdrCtas = 2,
  kHdrTile = 3,
  kHdrStatus = 4,
  kHdrBadIndex = 5,
  kHdrKind = 6,
  kHdrBatch = 7,
  kHdrMaxSegments = 8,
  kHdrSplits = 9,
  kHdrBalance = 10,  // 1: the plan used the descriptor's balance table (the decode follows its placement)
  kHdrWords = 16,
};

struct WsLayout {
  int64_t hdr, segs, req_tile_prefix, req_seg_begin, cta_seg_begin, req_done, total;
};

__host__ __device__ inline WsLayout ws_layout(int64_t batch, int64_t num_ctas, int64_t max_segments,
                                              int64_t num_kv_heads) {
  WsLayout L;
  L.hdr = 0;
  L.segs = kHdrWords;                       // int4 per segment, 64-byte aligned start
  L.req_tile_prefix = L.segs + 4 * max_segments;
  L.req_seg_begin = L.req_tile_prefix + batch + 1;
  L.cta_seg_begin = L.req_seg_begin + batch + 1;
  L.req_done = L.cta_seg_begin + num_ctas + 1;  // [batch][num_kv_heads] finished segments
  L.total = (L.req_done + batch * num_kv_heads + 3) / 4 * 4;
  return L;
}

// Record the first device-side data error (status word, then the offending index).
__device__ inline void record_status(int32_t* hdr, int32_t code, int32_t index) {
  if (atomicCAS(&hdr[kHdrStatus], DA_DEV_OK, code) == DA_DEV_OK) atomicExch(&hdr[kHdrBadIndex], index);
}

// ---- kernel parameter blocks -------------------------------------------------------------
struct PlanParams {
  const int32_t* seq_lens;
  int32_t* ws;
  int32_t batch, tile_tokens, width, max_segments, num_ctas, num_kv_heads;
  int64_t capacity_tokens;
  int32_t start_cost;  // dynamic plan: start units charged to every non-empty request
  const int32_t* balance;  // dynamic plan: balance table (weights and placement), or null
};

// Balance table: [magic, num_ctas, num_kv_heads, 0, weights[C], perm[Hkv][C]].
constexpr int32_t kBalanceMagic = 0x0DA0BA1A;
constexpr int32_t kBalanceMaxCtas = 2048;     // weighted ranges are kept in the planner's shared memory
constexpr int32_t kBalanceMaxWeight = 65536;
constexpr int kBalanceHeader = 4;

struct DecodeParams {
  const __nv_bfloat16* q;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* ws;
  float* partial_o;
  float* partial_lse;
  __nv_bfloat16* out;
  float* lse;
  int32_t batch, num_q_heads, num_kv_heads, group, page_size, max_pages_per_req, num_pages;
  int32_t tile_tokens, num_ctas, max_segments, kind;
  int64_t capacity_tokens;
  float scale_log2;  // scale * log2(e): scores are kept in base-2 units
  const float* k_scale;  // FP8 caches: per-KV-head dequantisation scales (else null)
  const float* v_scale;
  int32_t q_len;  // queries per request (1 = plain decode)
  int32_t full_rows;  // 1: q_len > 1 or G > 8: all 16 MMA rows carry (query, head) rows
  int32_t merge_in_decode;  // 1: the last CTA to finish a request's segment merges its partials
  int32_t stall_producer;   // failure-path test: the producer sends nothing, so every wait runs out
  uint64_t wait_limit_ns;   // limit of every pipeline wait
  int32_t out_f32;          // 1: every segment's result goes to the partials (the combine writes fp32 out)
  const int32_t* cta_perm;  // [Hkv][num_ctas]: the plan CTA block (x, g) runs, used when the plan took the
                            // balance table (header word kHdrBalance); null: block x runs CTA x
  int64_t* block_times;     // [Hkv][num_ctas][2]: start and end ns of every block, or null
};

struct CombineParams {
  const int32_t* ws;
  const float* partial_o;
  const float* partial_lse;
  __nv_bfloat16* out;
  float* lse;
  int32_t batch, num_q_heads, num_ctas, max_segments, num_kv_heads;
  int32_t out_f32;  // 1: out is fp32 and every request is written (one segment too)
};

struct AppendParams {
  const __nv_bfloat16* new_k;
  const __nv_bfloat16* new_v;
  const int32_t* block_table;
  const int32_t* seq_lens;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  int32_t* status;  // optional {code, index}
  int32_t batch, num_kv_heads, head_dim, page_size, max_pages_per_req, num_pages;
  int64_t capacity_tokens;
};

struct MergeParams {
  const __nv_bfloat16* part_out;  // [num_parts][rows][head_dim] (bf16 parts)
  const float* part_out_f32;      // or fp32 parts (exactly one of the two is set)
  const float* part_lse;          // [num_parts][rows]
  __nv_bfloat16* out;             // [rows][head_dim]
  float* lse;                     // [rows]
  int32_t num_parts;
  int64_t rows;
};

// One planned segment as the decode kernels walk it: request, token range [tok0, tok1)
// clipped to the request's length, and the length (bad lengths count as 0).  Every
// role of a decode CTA decodes a segment the same way, so all walk the same chunks.
struct SegmentInfo {
  int b, tok0, tok1, len;
  bool valid;
};

__device__ __forceinline__ bool segment_entry_valid(const DecodeParams& p, int4 sg) {
  return sg.x >= 0 && sg.x < p.batch && sg.z >= 0 && sg.w >= sg.z;
}

// The segment of plan entry sg, given its request's length as read from seq_lens (any value
// for an invalid entry).  Split from the loads so that a kernel can request them early.
__device__ __forceinline__ SegmentInfo make_segment(const DecodeParams& p, int4 sg, int L) {
  SegmentInfo r;
  r.b = sg.x;
  r.valid = segment_entry_valid(p, sg);
  if (!r.valid || L < 0 || (int64_t)L > p.capacity_tokens) L = 0;
  const int64_t t0 = (int64_t)sg.z * p.tile_tokens, t1 = min((int64_t)sg.w * p.tile_tokens, (int64_t)L);
  r.tok0 = (int)min(t0, (int64_t)L);
  r.tok1 = (int)t1;
  r.len = L;
  return r;
}

__device__ __forceinline__ SegmentInfo load_segment(const DecodeParams& p, const int4* segs, int s) {
  const int4 sg = segs[s];
  return make_segment(p, sg, segment_entry_valid(p, sg) ? p.seq_lens[sg.x] : 0);
}

// Host launchers (defined next to their kernels).
cudaError_t launch_plan_dynamic(const PlanParams& p, cudaStream_t stream);
cudaError_t launch_plan_static(const PlanParams& p, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams& p, int head_dim, const CUtensorMap maps[4], cudaStream_t stream);
cudaError_t launch_decode_fp8(const DecodeParams& p, int head_dim, const CUtensorMap maps[4], cudaStream_t stream);
cudaError_t launch_decode_fp8_tc(const DecodeParams& p, const CUtensorMap maps[4], cudaStream_t stream);
cudaError_t launch_combine(const CombineParams& p, int head_dim, cudaStream_t stream);
cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);
cudaError_t launch_merge(const MergeParams& p, int head_dim, cudaStream_t stream);

// Record a CUDA error for da_last_cuda_error() from code outside api.cu.
void set_last_cuda_error(cudaError_t e);

// ---- inline PTX ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- balance table in the decode kernels -----------------------------------------------
// The plan CTA that block (blockIdx.x, KV head blockIdx.y) runs if the plan took the balance
// table (read before the plan lands; an entry out of range keeps the block's own index).
__device__ __forceinline__ int placed_cta(const DecodeParams& p) {
  if (!p.cta_perm) return (int)blockIdx.x;
  const int c = __ldg(p.cta_perm + (int64_t)blockIdx.y * p.num_ctas + blockIdx.x);
  return c >= 0 && c < p.num_ctas ? c : (int)blockIdx.x;
}

// Thread 0: this block's start (t_start) and end times, when the descriptor asked for them.
__device__ __forceinline__ void record_block_times(const DecodeParams& p, uint64_t t_start) {
  if (p.block_times && threadIdx.x == 0) {
    int64_t* bt = p.block_times + ((int64_t)blockIdx.y * gridDim.x + blockIdx.x) * 2;
    bt[0] = (int64_t)t_start;
    bt[1] = (int64_t)global_timer_ns();
  }
}

// Bounded wait on an mbarrier phase.  Gives up (returns false) when *abort is
// set by another warp or after `limit_ns` of wall time, so no wait can spin
// forever.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort) return false;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > limit_ns) return false;
    }
  }
}

// Wait (at most limit_ns) for an mbarrier phase whatever the abort flag says: used to let
// the TMA copies a CTA requested land before the CTA exits, also after an abort.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0 && global_timer_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled TMA load global -> shared, completion counted on `bar` in bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + C, fp32 accumulate.  Only the
// upper 8 rows of A are used here (a1 = a3 = 0), so only d0, d1 are kept.
__device__ __forceinline__ void mma_bf16_upper(float& d0, float& d1, uint32_t a0, uint32_t a2, uint32_t b0,
                                               uint32_t b1) {
  float d2 = 0.f, d3 = 0.f;  // rows 8..15 of the tile: A is zero there
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// All 16 rows of A used (rows r: a0, a2; rows r + 8: a1, a3): d[0..1] row r, d[2..3] row r + 8.
__device__ __forceinline__ void mma_bf16_full(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_full(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Same with f16 operands (FP8 caches are widened to f16, exactly).
__device__ __forceinline__ void mma_f16_upper(float& d0, float& d1, uint32_t a0, uint32_t a2, uint32_t b0,
                                              uint32_t b1) {
  float d2 = 0.f, d3 = 0.f;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Programmatic dependent launch: wait for the previous kernel in the stream
// (no-op when the launch did not opt in).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace da

// decode.cu -- split-KV decode attention over a paged KV cache, sm_100a.
//
// "Tencent HPC lands in SGLang, challenging default inference kernels",
// section "Why Tencent HPC matters for online model serving": attention over
// each request's KV cache, with the cache work cut into uniform tiles that
// CTAs take from a plan rebuilt every step; a longer history means more
// cached data to read, so this kernel is bound by HBM reads of K and V.
//
// Grid (C, Hkv): CTA (c, g) walks the segments the plan gave CTA c, for KV
// head g.  Block = 4 consumer warps + 1 producer warp.
//
//   producer  One lane issues TMA tensor loads (128-byte swizzle) of K and V
//             chunks into a ring of shared-memory stages, each stage guarded
//             by a "full" mbarrier (transaction bytes) and an "empty" mbarrier
//             (one arrival per consumer warp).  A chunk is loaded as 64-row
//             boxes when a 64-token run sits inside one page, else as 16-row
//             boxes.  Page ids come from the block table 32 at a time.
//   consumers Warp w owns TPW consecutive tokens of each chunk (16 or 32) and
//             keeps its own online-softmax state for all G query heads of
//             the group:
//               S = Q . K^T with mma.m16n8k16 (rows = heads, the upper 8 of
//               the 16 MMA rows; n = tokens; k = head_dim), K read with
//               ldmatrix from the swizzled tile, two accumulator chains per
//               n-tile for instruction-level parallelism;
//               running max m, running sums, fp32 accumulator O += P . V with
//               P rounded to the MMA input type in registers and V read with
//               ldmatrix.trans; the sum of the rounded P comes from one more
//               MMA against a tile of ones; O is rescaled only when some row's
//               max moved.
//             At the end of a segment the four warp states are merged by
//             log-sum-exp through shared memory; the result goes to out/lse
//             (request with one segment) or to the segment's partial slot.
//
// Two cache formats share the kernel.  bf16: K/V rows feed a bf16 MMA directly.
// FP8 (E4M3 codes with one scale per KV head for K and for V): rows are half as
// wide (one 128-byte swizzle span at head_dim 128); K and V bytes are widened
// to f16 in registers (exact for every E4M3 value), q is converted bf16 -> f16
// (exact for normal-range values), P is rounded to f16, the MMA is f16 with
// fp32 accumulation, and the K scale is folded into the score scale and the V
// scale into the final normalisation.
//
// Every stage is 32 KB (K + V): 64 tokens of 256-byte rows (bf16, d 128) or
// 128 tokens of 128-byte rows (FP8 d 128, bf16 d 64); three stages per CTA and
// two CTAs per SM keep 192 KB of loads in flight per SM.
//
// Scores are kept in base-2 units (scale * log2 e), so exp is one ex2 and the
// natural-log lse is (m + log2 l) * ln 2.  Tokens past the end of a request
// inside a loaded chunk are masked to -inf; their V rows are zeroed in shared
// memory first, since unused cache slots may hold anything (NaN included).
#include <cuda_fp16.h>

#include <cfloat>

#include "da_internal.cuh"

namespace da {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

template <int D, bool FP8, bool MQ>
struct Cfg {
  static constexpr int kElemBytes = FP8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElemBytes;
  static_assert(kRowBytes % 128 == 0, "a row must be whole 128-byte swizzle spans");
  static constexpr int kHalves = kRowBytes / 128;            // 128-byte column blocks per row
  static constexpr int kBoxCols = 128 / kElemBytes;          // elements per TMA box row
  static constexpr int kNR = MQ ? 2 : 1;                     // MMA row halves used (upper 8 rows, or all 16)
  static constexpr int kTPW = (kRowBytes == 128 && !MQ) ? 32 : 16;  // tokens per consumer warp per chunk
  static constexpr int kChunk = kConsumerWarps * kTPW;       // tokens per stage
  static constexpr int kSub = kTPW / 16;                     // 16-token MMA pieces per warp
  static constexpr int kHalfStride = kChunk * 128;           // bytes of one 128-byte column block of a tile
  static constexpr int kTileBytes = kHalves * kHalfStride;   // one K (or V) chunk
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = (96 * 1024) / kStageBytes;  // a 96 KB ring per CTA
  // per-thread output columns: NG groups of GW consecutive columns, group gi at gi*4*GW + GW*tq
  static constexpr int kGW = FP8 ? 4 : 2;
  static constexpr int kNG = D / (4 * kGW);
  static constexpr int kSlotStride = D + (FP8 ? 16 : 8);     // floats per head row (bank-conflict free)
  static constexpr int kSlotFloats = 8 * kSlotStride;
  // shared memory map (offsets from a 1024-byte aligned base)
  static constexpr int kOffStages = 0;
  static constexpr int kOffSlots = kStages * kStageBytes;
  static constexpr int kOffML = kOffSlots + 3 * kSlotFloats * 4;        // [3][m, l_r, l_e][8] floats
  static constexpr int kOffBars = kOffML + 3 * 3 * 8 * 4;                // full[kStages], empty[kStages]
  static constexpr int kOffMeta = kOffBars + 2 * kStages * 8;            // int per stage
  static constexpr int kOffAbort = kOffMeta + kStages * 4;  // abort flag, then the "last segment" flag
  static constexpr int kBytes = kOffAbort + 16;
  static constexpr int kSmemRequest = kBytes + 1024;                     // slack for manual alignment
};

// Byte offset of (row, 16-byte column chunk) inside a TMA tile written with
// 128-byte swizzle: the chunk index is XORed with row % 8 inside each 128-byte
// row; column blocks of 128 bytes are stored one after the other.
template <int kHalfStride>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)((chunk >> 3) * kHalfStride + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// Four E4M3 codes c0..c3 (c0 in the low byte) -> two f16x2: lo = (c0, c1),
// hi = (c2, c3), low half first.  Exact: every E4M3 value is an f16 value.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t codes, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(codes));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}


// Merge every segment partial of request b for the rows of KV head g (G heads x
// q_len queries) into out/lse: LSE = M + ln sum_i exp(lse_i - M), out = sum_i
// exp(lse_i - LSE) o_i, fp32 in a fixed order.  Run by the four consumer warps of
// the CTA that finished the request's last segment; the partials of the other
// CTAs are read from L2 (ld.global.cg) after the acquire fence.
template <int D>
__device__ void merge_request_rows(const DecodeParams& p, int b, int g, int s0, int n, int qlen, int hq_rows,
                                   int warp, int lane) {
  constexpr int kPer = D / 32;
  const int rows = p.group * qlen;
  for (int R = warp; R < rows; R += 4) {
    const int qi = R / p.group, hj = R - qi * p.group;
    const int hrow = qi * p.num_q_heads + g * p.group + hj;
    const float* plse = p.partial_lse + (int64_t)s0 * hq_rows + hrow;
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) M = fmaxf(M, __ldcg(plse + (int64_t)i * hq_rows));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float total = -INFINITY;
    float acc[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
    if (M != -INFINITY) {
      float sum = 0.f;
      for (int i = lane; i < n; i += 32) sum += expf(__ldcg(plse + (int64_t)i * hq_rows) - M);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      total = M + logf(sum);
      const float* po = p.partial_o + ((int64_t)s0 * hq_rows + hrow) * D + lane * kPer;
#pragma unroll 8
      for (int i = 0; i < n; ++i) {
        const float wgt = expf(__ldcg(plse + (int64_t)i * hq_rows) - total);
        const float* src = po + (int64_t)i * hq_rows * D;
        if constexpr (kPer == 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
          acc[0] += wgt * v.x;
          acc[1] += wgt * v.y;
          acc[2] += wgt * v.z;
          acc[3] += wgt * v.w;
        } else {
          const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
          acc[0] += wgt * v.x;
          acc[1] += wgt * v.y;
        }
      }
    }
    __nv_bfloat16* dst = p.out + ((int64_t)b * hq_rows + hrow) * D + lane * kPer;
    if constexpr (kPer == 4)
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
    else
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0], acc[1]);
    if (lane == 0) p.lse[(int64_t)b * hq_rows + hrow] = total;
  }
}

#if DA_BF16_FFMA
// CUDA-core (FFMA) consumer for plain bf16 decode at head_dim 128, built only with
// -DDA_BF16_FFMA=1: the comparison point for the warp-level MMA consumer (same grid,
// producer, ring, plan and outputs).  Lane (h, qd) = (lane / 4, lane % 4) owns head h of
// the group and dims 32 qd .. 32 qd + 31.  Per token of its warp's 16 rows it dots q with
// the K row over its dims in fp32 (two shuffles finish the dot product), keeps head h's
// online softmax, and accumulates P.V over its 32 dims; P is not rounded.  The four warp
// states merge at segment end as in the MMA consumer.
template <typename C>
__device__ void ffma_consumer(const DecodeParams& p, uint8_t* smem, const int4* segs, const int32_t* rsb,
                              int32_t* hdr_w, uint32_t full0, uint32_t empty0, volatile int* meta,
                              volatile int* abort_flag, int seg_lo, int seg_hi, int g, int w, int lane) {
  constexpr int D = 128, TPW = C::kTPW, HS = C::kHalfStride;
  static_assert(C::kElemBytes == 2 && C::kRowBytes == 256 && TPW == 16, "bf16, head_dim 128");
  const int h = lane >> 2, qd = lane & 3;
  const bool live = h < p.group;
  float* slots = reinterpret_cast<float*>(smem + C::kOffSlots);
  float* ml = reinterpret_cast<float*>(smem + C::kOffML);
  int stage = 0;
  uint32_t phase = 0;
  for (int s = seg_lo; s < seg_hi; ++s) {
    const SegmentInfo si = load_segment(p, segs, s);
    if (!si.valid) continue;
    const int b = si.b;
    float qf[32];  // q of head h, dims 32 qd .., scaled to base-2 scores
    {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(
          p.q + ((int64_t)b * p.num_q_heads + (int64_t)g * p.group + (live ? h : 0)) * D + 32 * qd);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t u = live ? __ldg(src + j) : 0u;
        qf[2 * j] = bf16_lo_to_f32(u) * p.scale_log2;
        qf[2 * j + 1] = bf16_hi_to_f32(u) * p.scale_log2;
      }
    }
    float m = -INFINITY, l = 0.f, acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[e] = 0.f;
    for (int c0 = si.tok0; c0 < si.tok1; c0 += C::kChunk) {
      const bool got = mbar_wait_bounded(full0 + 8 * stage, phase, abort_flag, p.wait_limit_ns);
      if (!got && lane == 0) {
        if (!*abort_flag) record_status(hdr_w, DA_DEV_TIMEOUT, s);
        *abort_flag = 1;
      }
      const int n = got ? meta[stage] : 0;
      const int nw = min(max(n - TPW * w, 0), TPW);
      const uint8_t* kt = smem + C::kOffStages + stage * C::kStageBytes;
      const uint8_t* vt = kt + C::kTileBytes;
      if (nw > 0) {
        float sc[TPW];
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) {
          const int row = TPW * w + tt;
          float a = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 u = *reinterpret_cast<const uint4*>(kt + swz<HS>(row, 4 * qd + j));
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              a = fmaf(qf[8 * j + 2 * k], bf16_lo_to_f32(uw[k]), a);
              a = fmaf(qf[8 * j + 2 * k + 1], bf16_hi_to_f32(uw[k]), a);
            }
          }
          a += __shfl_xor_sync(0xffffffffu, a, 1);
          a += __shfl_xor_sync(0xffffffffu, a, 2);
          sc[tt] = tt < nw ? a : -INFINITY;  // rows past the loaded tokens may hold anything
        }
        float mx = sc[0];
#pragma unroll
        for (int tt = 1; tt < TPW; ++tt) mx = fmaxf(mx, sc[tt]);
        const float m_new = fmaxf(m, mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float corr = fast_exp2(m - m_use);
        l *= corr;
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] *= corr;
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) {
          if (tt >= nw) break;
          const float pt = fast_exp2(sc[tt] - m_use);
          l += pt;
          const int row = TPW * w + tt;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 u = *reinterpret_cast<const uint4*>(vt + swz<HS>(row, 4 * qd + j));
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              acc[8 * j + 2 * k] = fmaf(pt, bf16_lo_to_f32(uw[k]), acc[8 * j + 2 * k]);
              acc[8 * j + 2 * k + 1] = fmaf(pt, bf16_hi_to_f32(uw[k]), acc[8 * j + 2 * k + 1]);
            }
          }
        }
        m = m_new;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * stage);
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    // ---- merge the four warp states of this segment (head h, dims 32 qd ..)
    const bool direct = rsb[b + 1] - rsb[b] == 1 && !p.out_f32;
    if (w > 0) {
      float* slot = slots + (w - 1) * C::kSlotFloats + h * C::kSlotStride + 32 * qd;
#pragma unroll
      for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(slot + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
      if (qd == 0) {
        ml[(w - 1) * 24 + h] = m;
        ml[(w - 1) * 24 + 8 + h] = l;
      }
    }
    named_barrier_sync(1, kConsumerWarps * 32);
    if (w == 0) {
      float M = m, mw[3], lw[3];
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        mw[j] = ml[j * 24 + h];
        lw[j] = ml[j * 24 + 8 + h];
        M = fmaxf(M, mw[j]);
      }
      const bool empty = M == -INFINITY;
      const float f0 = empty ? 0.f : fast_exp2(m - M);
      float L = f0 * l, fw[3];
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        fw[j] = empty ? 0.f : fast_exp2(mw[j] - M);
        L += fw[j] * lw[j];
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const float lse_nat = L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float a = f0 * acc[e];
#pragma unroll
        for (int j = 0; j < 3; ++j) a += fw[j] * slots[j * C::kSlotFloats + h * C::kSlotStride + 32 * qd + e];
        acc[e] = a * inv;
      }
      if (live) {
        const int hrow = g * p.group + h;
        if (direct) {
          __nv_bfloat16* dst = p.out + ((int64_t)b * p.num_q_heads + hrow) * D + 32 * qd;
#pragma unroll
          for (int e = 0; e < 32; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e], acc[e + 1]);
          if (qd == 0) p.lse[(int64_t)b * p.num_q_heads + hrow] = lse_nat;
        } else {
          float* dst = p.partial_o + ((int64_t)s * p.num_q_heads + hrow) * D + 32 * qd;
#pragma unroll
          for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
          if (qd == 0) p.partial_lse[(int64_t)s * p.num_q_heads + hrow] = lse_nat;
        }
      }
    }
    named_barrier_sync(1, kConsumerWarps * 32);  // slots are free again
  }
}
#endif  // DA_BF16_FFMA

template <int D, bool FP8, bool MQ, bool MERGE>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap k64,
                  const __grid_constant__ CUtensorMap v64, const __grid_constant__ CUtensorMap k16,
                  const __grid_constant__ CUtensorMap v16) {
  using C = Cfg<D, FP8, MQ>;
  constexpr int kChunk = C::kChunk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  __shared__ unsigned long long s_t_start;

  // Prologue that does not depend on the plan: barriers and descriptor
  // prefetch overlap the planner kernel (programmatic dependent launch).
  const uint32_t full0 = sbase + C::kOffBars, empty0 = full0 + C::kStages * 8;
  volatile int* meta = reinterpret_cast<volatile int*>(smem + C::kOffMeta);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffAbort);
  const int placed = placed_cta(p);
  if (threadIdx.x == 0) {
    s_t_start = p.block_times ? global_timer_ns() : 0;
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kConsumerWarps && lane == 0) {
    prefetch_tensormap(&k64);
    prefetch_tensormap(&v64);
    prefetch_tensormap(&k16);
    prefetch_tensormap(&v16);
  }
  __syncthreads();

  // Stage `stage` <- K and V of tokens [c0, c0 + n) of one request, whose 16-token pieces sit
  // in pages pid[]; the stage's "full" barrier expects the bytes.  Lane 0 of the producer.
  constexpr int kPieces = kChunk / 16;
  auto issue_chunk = [&](int stage, int c0, int n, const int (&pid)[kPieces], bool ok, uint64_t policy) {
    const int P = p.page_size;
    meta[stage] = ok ? n : 0;
    // bytes: per 64-row sub-chunk, one 64-row box per column block when it sits in
    // one page, else one 16-row box per column block for each piece that holds tokens
    uint32_t bytes = 0;
    if (ok) {
#pragma unroll
      for (int j = 0; j < kChunk / 64; ++j) {
        if (64 * j >= n) break;
        const bool fast = ((c0 + 64 * j) % P) + 64 <= P;
        const int pieces = fast ? 4 : min(4, (n - 64 * j + 15) >> 4);
        bytes += (uint32_t)(pieces * 16 * 128 * C::kHalves * 2);
      }
    }
    const uint32_t full = full0 + 8 * stage;
    mbar_arrive_expect_tx(full, bytes);
    if (ok) {
      const uint32_t sk = sbase + C::kOffStages + stage * C::kStageBytes, sv = sk + C::kTileBytes;
#pragma unroll
      for (int j = 0; j < kChunk / 64; ++j) {
        if (64 * j >= n) break;
        const int tok = c0 + 64 * j;
        if ((tok % P) + 64 <= P) {
          const int row = (pid[4 * j] * p.num_kv_heads + g) * P + tok % P;
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {
            tma_load_2d(sk + h * C::kHalfStride + j * 64 * 128, &k64, h * C::kBoxCols, row, full, policy);
            tma_load_2d(sv + h * C::kHalfStride + j * 64 * 128, &v64, h * C::kBoxCols, row, full, policy);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (64 * j + 16 * i >= n) break;
            const int row = (pid[4 * j + i] * p.num_kv_heads + g) * P + (tok + 16 * i) % P;
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h) {
              const uint32_t off = h * C::kHalfStride + (64 * j + 16 * i) * 128;
              tma_load_2d(sk + off, &k16, h * C::kBoxCols, row, full, policy);
              tma_load_2d(sv + off, &v16, h * C::kBoxCols, row, full, policy);
            }
          }
        }
      }
    }
  };

  grid_dependency_wait();    // the plan is written by the previous kernel in the stream
  grid_dependents_launch();  // the combine kernel may be scheduled; it waits for this grid to finish

  const WsLayout WL = ws_layout(p.batch, p.num_ctas, p.max_segments, p.num_kv_heads);
  const int32_t* hdr = p.ws + WL.hdr;
  const int4* segs = reinterpret_cast<const int4*>(p.ws + WL.segs);
  const int32_t* rsb = p.ws + WL.req_seg_begin;
  const int32_t* csb = p.ws + WL.cta_seg_begin;
  int32_t* hdr_w = const_cast<int32_t*>(hdr);

  // The plan must match the descriptor this launch was given.  Which plan CTA this block runs:
  // its own index, or its place in the balance table if the plan took the table (both CTAs'
  // ranges are loaded with the header, so the choice adds no round trip).
  const int h_ctas = hdr[kHdrCtas], h_batch = hdr[kHdrBatch], h_ms = hdr[kHdrMaxSegments], h_kind = hdr[kHdrKind];
  const int own = blockIdx.x;
  const int h_segs = hdr[kHdrSegments], own_lo = csb[own], own_next = csb[own + 1];
  const int alt_lo = csb[placed], alt_next = csb[placed + 1];
  const bool balanced = hdr[kHdrBalance] == 1;
  const int cta = balanced ? placed : own;
  const int seg_lo = balanced ? alt_lo : own_lo, seg_next = balanced ? alt_next : own_next;
  if (h_ctas != p.num_ctas || h_batch != p.batch || h_ms != p.max_segments || h_kind != p.kind) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && g == 0) record_status(hdr_w, DA_DEV_BAD_PLAN, 0);
    record_block_times(p, s_t_start);
    return;
  }
  const int seg_hi = min(seg_next, min(h_segs, p.max_segments));
  if (MERGE && cta == 0) {
    // requests with no segment (length 0, or refused) get out = 0, lse = -inf here
    const int qlen0 = p.q_len > 1 ? p.q_len : 1;
    const int rows = p.group * qlen0, hq_rows0 = qlen0 * p.num_q_heads;
    for (int b = 0; b < p.batch; ++b) {
      if (rsb[b + 1] != rsb[b]) continue;
      for (int i = threadIdx.x; i < rows * (D / 8); i += kThreads) {
        const int R = i / (D / 8), c8 = i - R * (D / 8);
        const int hrow = (R / p.group) * p.num_q_heads + g * p.group + R % p.group;
        *reinterpret_cast<uint4*>(p.out + ((int64_t)b * hq_rows0 + hrow) * D + c8 * 8) = make_uint4(0, 0, 0, 0);
        if (c8 == 0) p.lse[(int64_t)b * hq_rows0 + hrow] = -INFINITY;
      }
    }
  }
  if (seg_lo < 0 || seg_lo >= seg_hi) {  // nothing planned for this CTA (uniform over the block)
    record_block_times(p, s_t_start);
    return;
  }

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------------ producer warp
    const uint64_t policy = policy_evict_first();
    const int P = p.page_size;
    int stage = 0;
    uint32_t phase = 0;
    int fills = 0;
    bool aborted = p.stall_producer != 0;  // failure-path test: send nothing
    for (int s = seg_lo; s < seg_hi && !aborted; ++s) {
      // first window of page ids, issued before (and independent of) the length load
      const int4 sg = segs[s];
      int win_base = INT_MIN / 2, win_val = -1;
      if (sg.x >= 0 && sg.x < p.batch && sg.z >= 0) {
        win_base = (int)((int64_t)sg.z * p.tile_tokens / P);
        const int lp = win_base + lane;
        win_val = lp < p.max_pages_per_req ? __ldg(p.block_table + (int64_t)sg.x * p.max_pages_per_req + lp) : -1;
      }
      const SegmentInfo si = load_segment(p, segs, s);
      if (!si.valid) continue;
      const int32_t* bt_row = p.block_table + (int64_t)si.b * p.max_pages_per_req;
      for (int c0 = si.tok0; c0 < si.tok1; c0 += kChunk) {
        const int n = min(kChunk, si.tok1 - c0);
        const int lp_first = c0 / P, lp_last = (c0 + n - 1) / P;
        if (lp_first < win_base || lp_last >= win_base + 32) {
          win_base = lp_first;
          const int lp = win_base + lane;
          win_val = lp < p.max_pages_per_req ? __ldg(bt_row + lp) : -1;
        }
        // page of every 16-row piece of the chunk (pieces past n are not loaded)
        int pid[kPieces];
        bool ok = true;
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          const int lp = (c0 + 16 * i) / P;
          pid[i] = __shfl_sync(0xffffffffu, win_val, (lp - win_base) & 31);
          if (16 * i < n) ok = ok && pid[i] >= 0 && pid[i] < p.num_pages;
        }
        // wait until the consumers have released this stage
        bool got = true;
        if (lane == 0) got = mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1, abort_flag, p.wait_limit_ns);
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          if (lane == 0) {
            if (!*abort_flag) record_status(hdr_w, DA_DEV_TIMEOUT, s);
            *abort_flag = 1;
          }
          aborted = true;
          break;
        }
        if (lane == 0) {
          if (!ok) record_status(hdr_w, DA_DEV_BAD_PAGE, si.b);
          issue_chunk(stage, c0, n, pid, ok, policy);
        }
        __syncwarp();
        ++fills;
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    // Drain: every stage's last fill must have landed before the CTA may exit (also after
    // an abort: the copies were requested, so they are waited for, within the limit).
    if (lane == 0) {
      for (int k = max(0, fills - C::kStages); k < fills; ++k)
        mbar_wait_drain(full0 + 8 * (k % C::kStages), (k / C::kStages) & 1, p.wait_limit_ns);
    }
    return;
  }

  // -------------------------------------------------------------------- consumer warps
#if DA_BF16_FFMA
  if constexpr (!FP8 && !MQ && !MERGE && D == 128) {
    ffma_consumer<C>(p, smem, segs, rsb, hdr_w, full0, empty0, meta, abort_flag, seg_lo, seg_hi, g, warp, lane);
    record_block_times(p, s_t_start);
    return;
  }
#endif
  constexpr int TPW = C::kTPW, SUB = C::kSub, HS = C::kHalfStride, NR = C::kNR;
  const int w = warp;
  const int r = lane >> 2;   // MMA row within a row half
  const int tq = lane & 3;   // thread within the quad
  // MMA row R = r + 8*hh (hh < NR) holds query qi = R / G of head hj = R % G of the group;
  // plain decode with G <= 8 uses only the upper 8 rows (R = r, the head).
  const int qlen = MQ ? p.q_len : 1;
  const int hq_rows = qlen * p.num_q_heads;  // output "heads" per request: q_len * Hq
  int qi[NR], hj[NR];
  bool live[NR];
#pragma unroll
  for (int hh = 0; hh < NR; ++hh) {
    if constexpr (MQ) {
      const int R = r + 8 * hh;
      qi[hh] = R / p.group;
      hj[hh] = R - qi[hh] * p.group;
      live[hh] = qi[hh] < qlen;
    } else {
      qi[hh] = 0;
      hj[hh] = r;
      live[hh] = r < p.group;
    }
  }
  float* slots = reinterpret_cast<float*>(smem + C::kOffSlots);
  float* ml = reinterpret_cast<float*>(smem + C::kOffML);
  int stage = 0;
  uint32_t phase = 0;

  // ldmatrix row addresses that do not depend on the chunk: lane i feeds row i%8
  // of matrix i/8.  Matrix order (tokens of a 16-token piece, 16-byte chunk):
  //   bf16 K  (0-7, c) (0-7, c+1) (8-15, c) (8-15, c+1)
  //   others  (0-7, c) (8-15, c) (0-7, c+1) (8-15, c+1)
  const int mat = lane >> 3, mrow = lane & 7;
  const int k_tok = TPW * w + (FP8 ? (mat & 1) * 8 : (mat >> 1) * 8) + mrow;
  const int k_chk = FP8 ? mat >> 1 : mat & 1;
  const int v_tok = TPW * w + (mat & 1) * 8 + mrow;
  const int v_chk = mat >> 1;
  const float k_scale = FP8 ? __ldg(p.k_scale + g) : 1.f;
  const float v_scale = FP8 ? __ldg(p.v_scale + g) : 1.f;
  const float score_scale = p.scale_log2 * k_scale;

  // D += A * B for one m16n8k16 tile; A rows r (a0, a2) and r + 8 (a1, a3).
  auto mma = [](float (&d)[2 * NR], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    if constexpr (NR == 1) {
      if constexpr (FP8) mma_f16_upper(d[0], d[1], a0, a2, b0, b1);
      else mma_bf16_upper(d[0], d[1], a0, a2, b0, b1);
    } else {
      if constexpr (FP8) mma_f16_full(d, a0, a1, a2, a3, b0, b1);
      else mma_bf16_full(d, a0, a1, a2, a3, b0, b1);
    }
  };

  for (int s = seg_lo; s < seg_hi; ++s) {
    const SegmentInfo si = load_segment(p, segs, s);
    if (!si.valid) continue;
    const int b = si.b;
    // tokens row hh may see: all L for plain decode; L - q_len + qi + 1 for query qi
    [[maybe_unused]] int vis[NR];
#pragma unroll
    for (int hh = 0; hh < NR; ++hh) vis[hh] = si.len - qlen + qi[hh] + 1;  // = len for plain decode

    // Q fragments, per row half; rows past the queries are zero.
    // bf16: k-block kk holds columns 16kk + 2tq + {0,1} and + 8.
    // FP8:  k-block kk holds columns 16kk + 4tq + {0,1} and {2,3}, as f16 (the
    //       order in which ldmatrix hands out the bytes of a K row).
    uint32_t qa[D / 16][NR][2];
#pragma unroll
    for (int hh = 0; hh < NR; ++hh) {
      const __nv_bfloat16* qh =
          p.q + (((int64_t)b * qlen + (live[hh] ? qi[hh] : 0)) * p.num_q_heads + (int64_t)g * p.group +
                 (live[hh] ? hj[hh] : 0)) * D;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        if constexpr (FP8) {
          const uint2 raw = live[hh] ? __ldg(reinterpret_cast<const uint2*>(qh) + 4 * kk + tq) : make_uint2(0, 0);
          qa[kk][hh][0] = pack_f16x2(bf16_lo_to_f32(raw.x), bf16_hi_to_f32(raw.x));
          qa[kk][hh][1] = pack_f16x2(bf16_lo_to_f32(raw.y), bf16_hi_to_f32(raw.y));
        } else {
          const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qh);
          qa[kk][hh][0] = live[hh] ? __ldg(q32 + kk * 8 + tq) : 0u;
          qa[kk][hh][1] = live[hh] ? __ldg(q32 + kk * 8 + 4 + tq) : 0u;
        }
      }
    }
    auto qA = [&](int kk, int part, int hh) -> uint32_t { return hh < NR ? qa[kk][hh < NR ? hh : 0][part] : 0u; };
    // lr: sum of the rounded weights that enter P.V (normalises O), kept as an
    //     MMA accumulator tile of P times ones (entries 2hh, 2hh+1 hold row half hh's sum);
    // l_e: per-thread sum of the unrounded fp32 weights (gives the log-sum-exp)
    float m[NR], l_e[NR];
    float lr[2 * NR];
#pragma unroll
    for (int hh = 0; hh < NR; ++hh) {
      m[hh] = -INFINITY;
      l_e[hh] = 0.f;
      lr[2 * hh] = lr[2 * hh + 1] = 0.f;
    }
    float o[D / 8][2 * NR];
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
#pragma unroll
      for (int e = 0; e < 2 * NR; ++e) o[i][e] = 0.f;

    for (int c0 = si.tok0; c0 < si.tok1; c0 += kChunk) {
      const bool got = mbar_wait_bounded(full0 + 8 * stage, phase, abort_flag, p.wait_limit_ns);
      if (!got && lane == 0) {
        if (!*abort_flag) record_status(hdr_w, DA_DEV_TIMEOUT, s);
        *abort_flag = 1;
      }
      const int n = got ? meta[stage] : 0;
      const int nw = min(max(n - TPW * w, 0), TPW);  // loaded tokens in this warp's rows
      const uint32_t sk = sbase + C::kOffStages + stage * C::kStageBytes, sv = sk + C::kTileBytes;
      if (nw > 0) {
        if (nw < TPW) {
          // zero V rows [nw, TPW) of this warp: stale or unused slots must not reach P.V
          uint8_t* vrows = smem + C::kOffStages + stage * C::kStageBytes + C::kTileBytes;
          for (int i = lane; i < (TPW - nw) * C::kHalves * 8; i += 32) {
            const int row = TPW * w + nw + i / (C::kHalves * 8);
            const int rem = i % (C::kHalves * 8);
            const int half = rem >> 3, chunk16 = rem & 7;
            *reinterpret_cast<uint4*>(vrows + half * HS + row * 128 + chunk16 * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        // tokens of this warp's rows that row half hh may see
        int lim[NR];
#pragma unroll
        for (int hh = 0; hh < NR; ++hh) {
          if constexpr (MQ) lim[hh] = min(nw, max(vis[hh] - c0 - TPW * w, 0));
          else lim[hh] = nw;  // a plain decode row sees every loaded token
        }
        // S = Q . K^T for this warp's tokens: n-tile nt = tokens [8nt, 8nt+8) of the
        // warp; two accumulator chains (even / odd k-blocks) per n-tile.
        float sc[2 * SUB][2][2 * NR];
#pragma unroll
        for (int nt = 0; nt < 2 * SUB; ++nt)
#pragma unroll
          for (int e = 0; e < 2 * NR; ++e) sc[nt][0][e] = sc[nt][1][e] = 0.f;
#pragma unroll
        for (int sp = 0; sp < SUB; ++sp) {
          const int ktok = k_tok + 16 * sp;
          if constexpr (FP8) {
#pragma unroll
            for (int kk = 0; kk < D / 16; kk += 2) {
              uint32_t r0, r1, r2, r3;  // (tile 0, kk) (tile 1, kk) (tile 0, kk+1) (tile 1, kk+1): 4 codes each
              ldmatrix_x4(sk + swz<HS>(ktok, kk + k_chk), r0, r1, r2, r3);
              uint32_t b00, b01, b10, b11, b20, b21, b30, b31;
              e4m3x4_to_f16x2x2(r0, b00, b01);
              e4m3x4_to_f16x2x2(r1, b10, b11);
              e4m3x4_to_f16x2x2(r2, b20, b21);
              e4m3x4_to_f16x2x2(r3, b30, b31);
              mma(sc[2 * sp][0], qA(kk, 0, 0), qA(kk, 0, 1), qA(kk, 1, 0), qA(kk, 1, 1), b00, b01);
              mma(sc[2 * sp + 1][0], qA(kk, 0, 0), qA(kk, 0, 1), qA(kk, 1, 0), qA(kk, 1, 1), b10, b11);
              mma(sc[2 * sp][1], qA(kk + 1, 0, 0), qA(kk + 1, 0, 1), qA(kk + 1, 1, 0), qA(kk + 1, 1, 1), b20, b21);
              mma(sc[2 * sp + 1][1], qA(kk + 1, 0, 0), qA(kk + 1, 0, 1), qA(kk + 1, 1, 0), qA(kk + 1, 1, 1), b30,
                  b31);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4(sk + swz<HS>(ktok, 2 * kk + k_chk), b0, b1, b2, b3);
              mma(sc[2 * sp][kk & 1], qA(kk, 0, 0), qA(kk, 0, 1), qA(kk, 1, 0), qA(kk, 1, 1), b0, b1);
              mma(sc[2 * sp + 1][kk & 1], qA(kk, 0, 0), qA(kk, 0, 1), qA(kk, 1, 0), qA(kk, 1, 1), b2, b3);
            }
          }
        }
        // scale to base 2, mask what a row may not see (only in a partial chunk or at
        // a query's causal edge), online softmax update per row half
        float x[2 * SUB][NR][2];
#pragma unroll
        for (int nt = 0; nt < 2 * SUB; ++nt)
#pragma unroll
          for (int hh = 0; hh < NR; ++hh)
#pragma unroll
            for (int e = 0; e < 2; ++e) x[nt][hh][e] = (sc[nt][0][2 * hh + e] + sc[nt][1][2 * hh + e]) * score_scale;
        bool partial = lim[0] < TPW;
        if constexpr (NR == 2) partial = partial || lim[1] < TPW;
        if (__any_sync(0xffffffffu, partial)) {
#pragma unroll
          for (int nt = 0; nt < 2 * SUB; ++nt)
#pragma unroll
            for (int hh = 0; hh < NR; ++hh)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                if (8 * nt + 2 * tq + e >= lim[hh]) x[nt][hh][e] = -INFINITY;
        }
        float corr[NR], m_use[NR];
        bool moved = false;
#pragma unroll
        for (int hh = 0; hh < NR; ++hh) {
          float mx = -INFINITY;
#pragma unroll
          for (int nt = 0; nt < 2 * SUB; ++nt) mx = fmaxf(mx, fmaxf(x[nt][hh][0], x[nt][hh][1]));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          const float m_new = fmaxf(m[hh], mx);
          m_use[hh] = m_new == -INFINITY ? 0.f : m_new;
          corr[hh] = fast_exp2(m[hh] - m_use[hh]);
          moved = moved || corr[hh] != 1.f;
          m[hh] = m_new;
        }
        // P fragments (A operand of P.V): rows r (a0, a2) and r + 8 (a1, a3),
        // tokens 0-7 of the piece in a0/a1 and 8-15 in a2/a3
        uint32_t pa[SUB][4];
#pragma unroll
        for (int sp = 0; sp < SUB; ++sp) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (hh >= NR) {
              pa[sp][hh] = pa[sp][2 + hh] = 0u;
              continue;
            }
            const int h2 = hh < NR ? hh : 0;
            const float p00 = fast_exp2(x[2 * sp][h2][0] - m_use[h2]), p01 = fast_exp2(x[2 * sp][h2][1] - m_use[h2]);
            const float p10 = fast_exp2(x[2 * sp + 1][h2][0] - m_use[h2]);
            const float p11 = fast_exp2(x[2 * sp + 1][h2][1] - m_use[h2]);
            if constexpr (FP8) {
              pa[sp][hh] = pack_f16x2(p00, p01);
              pa[sp][2 + hh] = pack_f16x2(p10, p11);
            } else {
              pa[sp][hh] = pack_bf16x2(p00, p01);
              pa[sp][2 + hh] = pack_bf16x2(p10, p11);
            }
            l_e[h2] = (sp == 0 ? l_e[h2] * corr[h2] : l_e[h2]) + ((p00 + p01) + (p10 + p11));
          }
        }
        if (__any_sync(0xffffffffu, moved)) {  // some row's running max moved
#pragma unroll
          for (int hh = 0; hh < NR; ++hh) {
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
              o[i][2 * hh] *= corr[hh];
              o[i][2 * hh + 1] *= corr[hh];
            }
            lr[2 * hh] *= corr[hh];
            lr[2 * hh + 1] *= corr[hh];
          }
        }
        // the sum of the rounded weights, as the tensor core sees them: P times a
        // column block of ones (every column of the tile holds the row sum)
        constexpr uint32_t kOnes = FP8 ? 0x3C003C00u : 0x3F803F80u;
#pragma unroll
        for (int sp = 0; sp < SUB; ++sp) mma(lr, pa[sp][0], pa[sp][1], pa[sp][2], pa[sp][3], kOnes, kOnes);
        // O += P . V, one k-step of 16 tokens per piece
#pragma unroll
        for (int sp = 0; sp < SUB; ++sp) {
          const int vtok = v_tok + 16 * sp;
          if constexpr (FP8) {
            // ldmatrix.trans hands each thread, per matrix, the code pairs (t0: d, d+1)
            // and (t1: d, d+1) as bytes 0..3; one byte permute to (0, 2, 1, 3) gives
            // column d's pair (t0, t1) and column d+1's pair.  Tile 2c + e holds
            // columns 16c + 2j + e.
#pragma unroll
            for (int c = 0; c < D / 16; c += 2) {
              uint32_t r0, r1, r2, r3;  // (tok 0-7, c) (tok 8-15, c) (tok 0-7, c+1) (tok 8-15, c+1)
              ldmatrix_x4_trans(sv + swz<HS>(vtok, c + v_chk), r0, r1, r2, r3);
              uint32_t e0, o0, e1, o1, e2, o2, e3, o3;
              e4m3x4_to_f16x2x2(__byte_perm(r0, 0, 0x3120), e0, o0);
              e4m3x4_to_f16x2x2(__byte_perm(r1, 0, 0x3120), e1, o1);
              e4m3x4_to_f16x2x2(__byte_perm(r2, 0, 0x3120), e2, o2);
              e4m3x4_to_f16x2x2(__byte_perm(r3, 0, 0x3120), e3, o3);
              mma(o[2 * c], pa[sp][0], pa[sp][1], pa[sp][2], pa[sp][3], e0, e1);
              mma(o[2 * c + 1], pa[sp][0], pa[sp][1], pa[sp][2], pa[sp][3], o0, o1);
              mma(o[2 * c + 2], pa[sp][0], pa[sp][1], pa[sp][2], pa[sp][3], e2, e3);
              mma(o[2 * c + 3], pa[sp][0], pa[sp][1], pa[sp][2], pa[sp][3], o2, o3);
            }
          } else {
#pragma unroll
            for (int np = 0; np < D / 16; ++np) {
              uint32_t v0, v1, v2, v3;
              ldmatrix_x4_trans(sv + swz<HS>(vtok, 2 * np + v_chk), v0, v1, v2, v3);
              mma(o[2 * np], pa[sp][0], pa[sp][1], pa[sp][2], pa[sp][3], v0, v1);
              mma(o[2 * np + 1], pa[sp][0], pa[sp][1], pa[sp][2], pa[sp][3], v2, v3);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * stage);
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1;
      }
    }

    // ---- merge the four warp states of this segment, one row half at a time
    const int nseg_b = rsb[b + 1] - rsb[b];
    const bool direct = nseg_b == 1 && !p.out_f32;  // fp32 output: the combine writes every request
#pragma unroll
    for (int hh = 0; hh < NR; ++hh) {
      // regroup this thread's columns: og[gi][j] is column gi*4*GW + GW*tq + j
      constexpr int GW = C::kGW, NG = C::kNG;
      float og[NG][GW];
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        if constexpr (FP8) {  // tiles 2gi (even columns) and 2gi+1 (odd columns) of chunk gi
          og[gi][0] = o[2 * gi][2 * hh];
          og[gi][1] = o[2 * gi + 1][2 * hh];
          og[gi][2] = o[2 * gi][2 * hh + 1];
          og[gi][3] = o[2 * gi + 1][2 * hh + 1];
        } else {
          og[gi][0] = o[gi][2 * hh];
          og[gi][1] = o[gi][2 * hh + 1];
        }
      }
      const float l_r = lr[2 * hh];  // already the full row sum over the warp's tokens
      float le = l_e[hh];
      le += __shfl_xor_sync(0xffffffffu, le, 1);
      le += __shfl_xor_sync(0xffffffffu, le, 2);
      if (w > 0) {
        float* slot = slots + (w - 1) * C::kSlotFloats + r * C::kSlotStride + GW * tq;
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) {
          if constexpr (GW == 4)
            *reinterpret_cast<float4*>(slot + 16 * gi) = make_float4(og[gi][0], og[gi][1], og[gi][2], og[gi][3]);
          else
            *reinterpret_cast<float2*>(slot + 8 * gi) = make_float2(og[gi][0], og[gi][1]);
        }
        if (tq == 0) {
          ml[(w - 1) * 24 + r] = m[hh];
          ml[(w - 1) * 24 + 8 + r] = l_r;
          ml[(w - 1) * 24 + 16 + r] = le;
        }
      }
      named_barrier_sync(1, kConsumerWarps * 32);
      if (w == 0) {
        float mw[3], lrw[3], lew[3];
        float M = m[hh];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          mw[j] = ml[j * 24 + r];
          lrw[j] = ml[j * 24 + 8 + r];
          lew[j] = ml[j * 24 + 16 + r];
          M = fmaxf(M, mw[j]);
        }
        const bool empty = M == -INFINITY;
        const float f0 = empty ? 0.f : fast_exp2(m[hh] - M);
        float fw[3];
        float Lr = f0 * l_r, Le = f0 * le;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          fw[j] = empty ? 0.f : fast_exp2(mw[j] - M);
          Lr += fw[j] * lrw[j];
          Le += fw[j] * lew[j];
        }
        const float inv = Lr > 0.f ? v_scale / Lr : 0.f;
        const float lse_nat = Le > 0.f ? (M + log2f(Le)) * 0.69314718055994530942f : -INFINITY;
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) {
          float a[GW];
#pragma unroll
          for (int e = 0; e < GW; ++e) a[e] = f0 * og[gi][e];
#pragma unroll
          for (int j = 0; j < 3; ++j) {
            const float* src = slots + j * C::kSlotFloats + r * C::kSlotStride + gi * 4 * GW + GW * tq;
#pragma unroll
            for (int e = 0; e < GW; ++e) a[e] += fw[j] * src[e];
          }
#pragma unroll
          for (int e = 0; e < GW; ++e) og[gi][e] = a[e] * inv;
        }
        if (live[hh]) {
          // output row: query qi, head g*G + hj, i.e. "head" qi*Hq + g*G + hj of q_len*Hq
          const int hrow = qi[hh] * p.num_q_heads + g * p.group + hj[hh];
          if (direct) {
            __nv_bfloat16* dst = p.out + ((int64_t)b * hq_rows + hrow) * D + GW * tq;
#pragma unroll
            for (int gi = 0; gi < NG; ++gi) {
              if constexpr (GW == 4)
                *reinterpret_cast<uint2*>(dst + 16 * gi) =
                    make_uint2(pack_bf16x2(og[gi][0], og[gi][1]), pack_bf16x2(og[gi][2], og[gi][3]));
              else
                *reinterpret_cast<uint32_t*>(dst + 8 * gi) = pack_bf16x2(og[gi][0], og[gi][1]);
            }
            if (tq == 0) p.lse[(int64_t)b * hq_rows + hrow] = lse_nat;
          } else {
            float* dst = p.partial_o + ((int64_t)s * hq_rows + hrow) * D + GW * tq;
#pragma unroll
            for (int gi = 0; gi < NG; ++gi) {
              if constexpr (GW == 4)
                *reinterpret_cast<float4*>(dst + 16 * gi) = make_float4(og[gi][0], og[gi][1], og[gi][2], og[gi][3]);
              else
                *reinterpret_cast<float2*>(dst + 8 * gi) = make_float2(og[gi][0], og[gi][1]);
            }
            if (tq == 0) p.partial_lse[(int64_t)s * hq_rows + hrow] = lse_nat;
          }
        }
      }
      named_barrier_sync(1, kConsumerWarps * 32);  // slots are free again
    }
    // ---- the CTA that finishes a split request's last segment merges its partials
    if (MERGE && !direct) {
      volatile int* last_flag = abort_flag + 1;
      if (w == 0) {
        __threadfence();  // this segment's partials are visible before the count moves
        __syncwarp();
        if (lane == 0) {
          const int prev = atomicAdd(const_cast<int32_t*>(p.ws) + WL.req_done + (int64_t)b * p.num_kv_heads + g, 1);
          *last_flag = prev == nseg_b - 1;
        }
      }
      named_barrier_sync(1, kConsumerWarps * 32);
      if (*last_flag) {
        __threadfence();  // acquire: the other CTAs' partials
        merge_request_rows<D>(p, b, g, rsb[b], nseg_b, qlen, hq_rows, w, lane);
      }
    }
  }
  record_block_times(p, s_t_start);  // thread 0 is a consumer: every segment of the block is done
}

template <int D, bool FP8, bool MQ, bool MERGE>
cudaError_t launch_decode_d(const DecodeParams& p, const CUtensorMap maps[4], cudaStream_t stream) {
  using C = Cfg<D, FP8, MQ>;
  static_assert(C::kSmemRequest * 2 <= 227 * 1024, "two CTAs per SM must fit");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool configured[64] = {false};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(decode_kernel<D, FP8, MQ, MERGE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemRequest);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.num_ctas, (unsigned)p.num_kv_heads, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemRequest;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<D, FP8, MQ, MERGE>, p, maps[0], maps[1], maps[2], maps[3]);
}

template <int D, bool FP8>
cudaError_t launch_variant(const DecodeParams& p, const CUtensorMap maps[4], cudaStream_t stream) {
  const bool mq = p.full_rows != 0, merge = p.merge_in_decode != 0;
  if (mq) return merge ? launch_decode_d<D, FP8, true, true>(p, maps, stream)
                       : launch_decode_d<D, FP8, true, false>(p, maps, stream);
  return merge ? launch_decode_d<D, FP8, false, true>(p, maps, stream)
               : launch_decode_d<D, FP8, false, false>(p, maps, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int head_dim, const CUtensorMap maps[4], cudaStream_t stream) {
  if (head_dim == 128) return launch_variant<128, false>(p, maps, stream);
  if (head_dim == 64) return launch_variant<64, false>(p, maps, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_fp8(const DecodeParams& p, int head_dim, const CUtensorMap maps[4], cudaStream_t stream) {
  if (head_dim == 128) return launch_variant<128, true>(p, maps, stream);
  return cudaErrorInvalidValue;
}

}  // namespace da

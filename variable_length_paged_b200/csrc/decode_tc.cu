// decode_tc.cu -- split-KV decode attention over an FP8 (E4M3) paged KV cache
// on the 5th-generation tensor cores: tcgen05.mma with accumulators in tensor
// memory (TMEM), operands straight from the TMA-filled shared-memory rings.
//
// "Tencent HPC lands in SGLang, challenging default inference kernels",
// sections "Why Tencent HPC matters for online model serving" (attention over
// each request's cached history, the work cut into uniform tiles spread over
// CTAs by a per-step plan) and "What the 48.8% TPOT claim does not prove"
// (cache precision is one of the settings that decide the result).
//
// Same plan, workspace, partials and outputs as decode.cu; used for plain
// decode (one query per request, at most 8 query heads per KV head, head_dim
// 128).  CTA (c, g) walks the segments of CTA c for KV head g, 128 tokens per
// chunk.  The tokens of a chunk are the 128 lanes of the MMA (M = 128):
//
//   S^T = K . [q_hi | q_lo]^T      A = K tile (K-major, 128-byte swizzle, as TMA
//                                  wrote it), B = 16 rows of E4M3 q: rows 0-7 the
//                                  hi terms of the G heads, rows 8-15 the lo
//                                  terms; N = 16, four k = 32 steps over head_dim
//   O^T = V^T . [P_hi | P_lo]^T    A = the same V tile read M(dim)-major, B = the
//                                  weights of the chunk's 128 tokens, 16 bytes per
//                                  token (hi terms of 8 heads, then lo terms);
//                                  N = 16, four k = 32 steps over the tokens
//
// q (times a power of two per head) and P' (= 2^8 P) enter as two E4M3 terms
// each, hi = e4m3(x) and lo = e4m3(x - hi), which keep 8 significant bits, the
// precision of bf16; every product of two E4M3 values is exact in the fp32
// accumulator.  P' is taken relative to each chunk's own maximum (floored at
// the running maximum minus kFloor), so that a chunk's largest weight enters
// as 2^8 and the small weights never fall into E4M3's coarse subnormals; the
// fp32 state (O and the weight sums) is rescaled to each chunk's reference.
//
// Warps: 0-3 softmax (thread t = token t of a chunk for S, dim t for O; warp w
// reads TMEM lanes 32w..32w+31; each warp announces its weights of a chunk on an
// mbarrier), 4 TMA producer, 5 MMA issuer (one thread: the score MMA of a chunk as
// soon as its K tile has landed, its P.V as soon as all four warps' weights are in).
//
// K and V of a chunk are requested together but held in separate rings: a K
// tile is read once, by the score MMA, and its slot is handed back when that
// MMA completes (~2.3 us after the request under load); a V tile waits for the
// softmax and the P.V MMA as well (~4 us).  Two K slots and four V slots (96 KB,
// the same as three joint stages) keep up to four chunks in flight where joint
// stages allowed three, with the K ring no longer held through the softmax.
//
// TMEM: 64 columns = S[2] and O[2] (16 fp32 columns each), double buffered so
// the tensor core computes chunk i+1's scores while the softmax warps work on
// chunk i.  The q tile is double buffered too: segment j+1's tile is written when
// segment j starts, so the MMA thread runs on across segment boundaries.  Every
// wait is bounded (DecodeParams::wait_limit_ns); TMEM is freed on every path out.
#include <cuda_fp16.h>

#include <cfloat>
#include <climits>

#include "da_internal.cuh"

namespace da {
namespace {

constexpr int kD = 128;               // head_dim: one 128-byte row of E4M3 codes
constexpr int kChunk = 128;           // tokens per chunk = lanes of one MMA
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreadsTc = 6 * 32;
constexpr int kKSlots = 2;            // K tiles, each freed when its chunk's score MMA completes
constexpr int kVSlots = 4;            // V tiles, each freed when its chunk's P.V MMA completes
constexpr int kTileBytes = kChunk * 128;  // K (or V) of one chunk: 16 KB
constexpr uint32_t kTmemCols = 64;    // S[2] at columns 0, 16; O[2] at 32, 48
constexpr float kPShift = 8.f;        // P' = 2^8 P
constexpr float kFloor = 40.f;        // a chunk's reference stays within 2^40 of the running max

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kOffK = 0;                          // [kKSlots][128 tokens x 128 B], 128-byte swizzle
constexpr int kOffV = kOffK + kKSlots * kTileBytes;  // [kVSlots][128 tokens x 128 B], 128-byte swizzle
constexpr int kOffQ8 = kOffV + kVSlots * kTileBytes;  // [2][16 rows x 128 B], 128-byte swizzle (1024-aligned)
constexpr int kOffP = kOffQ8 + 2 * 2048;         // [2][128 tokens][16 B]
constexpr int kOffRed = kOffP + 2 * 2048;        // [2][4 warps][8] floats
constexpr int kOffRowScale = kOffRed + 2 * 32 * 4;  // [2][8] floats
constexpr int kOffBars = kOffRowScale + 2 * 8 * 4;
// mbarriers: k_full[2], k_empty[2], v_full[4], v_empty[4], s_full[2], s_free[2], o_full[2],
// q_full[2], done (MMA thread), p_full[2] (the four softmax warps' weights of a chunk are written)
constexpr int kBarKFull = 0, kBarKEmpty = 2, kBarVFull = 4, kBarVEmpty = 8, kBarSFull = 12, kBarSFree = 14,
              kBarOFull = 16, kBarQFull = 18, kBarDone = 20, kBarPFull = 21, kNumBars = 23;
constexpr int kOffMeta = kOffBars + kNumBars * 8;  // loaded tokens of the chunk in each V slot
constexpr int kOffFlags = kOffMeta + kVSlots * 4;  // abort flag, TMEM base address
constexpr int kBytesTc = kOffFlags + 16;
constexpr int kSmemTc = kBytesTc + 1024;  // slack for the manual 1024-byte alignment
static_assert(kOffQ8 % 1024 == 0 && kOffP % 16 == 0 && kOffBars % 8 == 0, "alignment");

// Instruction descriptor of kind::f8f6f4: E4M3 x E4M3 -> fp32, M = 128, N = 16.
// Bits: [4,6) D format (1 = f32), [7,10) A format, [10,13) B format (0 = E4M3),
// 15 A major, 16 B major (0 = K-major, 1 = MN-major), [17,23) N / 8, [24,29) M / 16.
constexpr uint32_t kIdescS = (1u << 4) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 15) | (1u << 16);

// Shared-memory matrix descriptor: start address, leading and stride byte offsets
// (all in 16-byte units), version 1, layout (2 = 128-byte swizzle, 0 = none).
//   K tile, Q8 (K-major, 128-byte swizzle): 8-row groups 1024 B apart (stride offset).
//   V tile read dim-major (MN-major, 128-byte swizzle): 8-token groups 1024 B apart; the
//     128 dims are one swizzle atom, so the other offset is unused and set equal.
//   P' (MN-major, no swizzle): 8-token core matrices of 16 B rows, 128 B apart; N = 16
//     is one core matrix wide, so the other offset is unused and set equal.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46) | ((uint64_t)layout << 61);
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A * B; issued by one thread.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane; the wait is tied to the
// registers so that no use can be scheduled before the load has landed.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])::"memory");
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// f16x2 -> two E4M3 codes in the low 16 bits (low half -> low byte), nearest even, saturating.
__device__ __forceinline__ uint32_t f16x2_to_e4m3x2(uint32_t h) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(r) : "r"(h));
  return r;
}

// Two E4M3 codes (low byte first) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t c) {
  uint32_t r;
  asm("{\n\t.reg .b16 l;\n\tcvt.u16.u32 l, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t}" : "=r"(r) : "r"(c));
  return r;
}

// x (f16x2) as hi + lo, two E4M3 terms per element (16-bit code pairs).
__device__ __forceinline__ void split_e4m3x2(uint32_t x, uint32_t& hi, uint32_t& lo) {
  hi = f16x2_to_e4m3x2(x);
  const uint32_t back = e4m3x2_to_f16x2(hi);
  uint32_t rem;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(rem) : "r"(x), "r"(back));
  lo = f16x2_to_e4m3x2(rem);
}

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait on an mbarrier phase for at most `limit_ns`, whatever the abort flag says
// (used to drain the tensor core before TMEM is freed).
__device__ __forceinline__ bool mbar_wait_timeout(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0 && global_timer_ns() - t0 > limit_ns) return false;
  }
}

// Reduce 8 per-thread values over the 128 softmax threads (max or sum); every
// thread gets all 8 results.  Inside a warp: halve the set at each of three
// exchanges (lane bit 4, 3, 2 picks the half kept), then two plain steps, so lane
// l holds value (l >> 2) & 7 over the warp; four warps meet in shared memory.
// `red` is double buffered by the caller's call count, so one barrier per call.
template <bool kMax>
__device__ __forceinline__ void reduce8(const float (&v)[8], float (&out)[8], float* red, int warp, int lane) {
  auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
  float a[4], c[2];
  const bool u4 = lane & 16, u3 = lane & 8, u2 = lane & 4;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float keep = u4 ? v[4 + k] : v[k], give = u4 ? v[k] : v[4 + k];
    a[k] = op(keep, __shfl_xor_sync(0xffffffffu, give, 16));
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float keep = u3 ? a[2 + k] : a[k], give = u3 ? a[k] : a[2 + k];
    c[k] = op(keep, __shfl_xor_sync(0xffffffffu, give, 8));
  }
  float x = op(u2 ? c[1] : c[0], __shfl_xor_sync(0xffffffffu, u2 ? c[0] : c[1], 4));
  x = op(x, __shfl_xor_sync(0xffffffffu, x, 2));
  x = op(x, __shfl_xor_sync(0xffffffffu, x, 1));
  if ((lane & 3) == 0) red[warp * 8 + (lane >> 2)] = x;
  named_barrier_sync(1, kSoftmaxWarps * 32);
  const float4* r4 = reinterpret_cast<const float4*>(red);
#pragma unroll
  for (int h = 0; h < 8; h += 4) {
    float4 s = r4[h / 4];
#pragma unroll
    for (int w = 1; w < kSoftmaxWarps; ++w) {
      const float4 t = r4[w * 2 + h / 4];
      s = make_float4(op(s.x, t.x), op(s.y, t.y), op(s.z, t.z), op(s.w, t.w));
    }
    out[h] = s.x;
    out[h + 1] = s.y;
    out[h + 2] = s.z;
    out[h + 3] = s.w;
  }
}

__global__ void __launch_bounds__(kThreadsTc, 2)
    decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap k64,
                     const __grid_constant__ CUtensorMap v64, const __grid_constant__ CUtensorMap k16,
                     const __grid_constant__ CUtensorMap v16) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  __shared__ unsigned long long s_t_start;
  const int placed = placed_cta(p);  // the plan CTA this block runs if the plan took the balance table
  const uint32_t bars = sbase + kOffBars;
  auto bar = [bars](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  volatile int* meta = reinterpret_cast<volatile int*>(smem + kOffMeta);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffFlags);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffFlags + 4);

  if (threadIdx.x == 0) {
    s_t_start = p.block_times ? global_timer_ns() : 0;
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);  // released by the tensor core (commit after S)
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);  // released by the tensor core (commit after P.V)
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(bar(kBarSFull + j), 1);
      mbar_init(bar(kBarSFree + j), kSoftmaxWarps);
      mbar_init(bar(kBarOFull + j), 1);
    }
    mbar_init(bar(kBarQFull), kSoftmaxWarps);
    mbar_init(bar(kBarQFull + 1), kSoftmaxWarps);
    mbar_init(bar(kBarDone), 1);
    mbar_init(bar(kBarPFull), kSoftmaxWarps);
    mbar_init(bar(kBarPFull + 1), kSoftmaxWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&k64);
    prefetch_tensormap(&v64);
    prefetch_tensormap(&k16);
    prefetch_tensormap(&v16);
  }
  __syncthreads();

  // K slot ks <- K codes, V slot vs <- V codes of tokens [c0, c0 + n) of one request, whose
  // 16-token pieces sit in pages pid[]; each slot's "full" barrier expects its bytes.  Both
  // tiles of a chunk are requested together.  Lane 0 of the producer.
  constexpr int kPieces = kChunk / 16;
  auto issue_chunk = [&](int ks, int vs, int c0, int n, const int (&pid)[kPieces], bool ok, uint64_t policy) {
    const int P = p.page_size;
    meta[vs] = ok ? n : 0;
    uint32_t bytes = 0;  // of one tile
    if (ok) {
#pragma unroll
      for (int j = 0; j < kChunk / 64; ++j) {
        if (64 * j >= n) break;
        const bool fast = ((c0 + 64 * j) % P) + 64 <= P;
        const int pieces = fast ? 4 : min(4, (n - 64 * j + 15) >> 4);
        bytes += (uint32_t)(pieces * 16 * 128);
      }
    }
    const uint32_t kfull = bar(kBarKFull + ks), vfull = bar(kBarVFull + vs);
    mbar_arrive_expect_tx(kfull, bytes);
    mbar_arrive_expect_tx(vfull, bytes);
    if (ok) {
      const uint32_t sk = sbase + kOffK + ks * kTileBytes, sv = sbase + kOffV + vs * kTileBytes;
#pragma unroll
      for (int j = 0; j < kChunk / 64; ++j) {
        if (64 * j >= n) break;
        const int tok = c0 + 64 * j;
        if ((tok % P) + 64 <= P) {
          const int row = (pid[4 * j] * p.num_kv_heads + g) * P + tok % P;
          tma_load_2d(sk + j * 64 * 128, &k64, 0, row, kfull, policy);
          tma_load_2d(sv + j * 64 * 128, &v64, 0, row, vfull, policy);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (64 * j + 16 * i >= n) break;
            const int row = (pid[4 * j + i] * p.num_kv_heads + g) * P + (tok + 16 * i) % P;
            const uint32_t off = (64 * j + 16 * i) * 128;
            tma_load_2d(sk + off, &k16, 0, row, kfull, policy);
            tma_load_2d(sv + off, &v16, 0, row, vfull, policy);
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
  const int32_t* csb = p.ws + WL.cta_seg_begin;
  int32_t* hdr_w = const_cast<int32_t*>(hdr);
  const int h_ctas = hdr[kHdrCtas], h_batch = hdr[kHdrBatch], h_ms = hdr[kHdrMaxSegments], h_kind = hdr[kHdrKind];
  const int own = blockIdx.x;
  const int h_segs = hdr[kHdrSegments], own_lo = csb[own], own_next = csb[own + 1];
  const int alt_lo = csb[placed], alt_next = csb[placed + 1];
  const bool balanced = hdr[kHdrBalance] == 1;  // the plan took the balance table: follow its placement
  const int seg_lo = balanced ? alt_lo : own_lo, seg_next = balanced ? alt_next : own_next;
  if (h_ctas != p.num_ctas || h_batch != p.batch || h_ms != p.max_segments || h_kind != p.kind) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && g == 0) record_status(hdr_w, DA_DEV_BAD_PLAN, 0);
    record_block_times(p, s_t_start);
    return;  // before TMEM is allocated
  }
  const int seg_hi = min(seg_next, min(h_segs, p.max_segments));
  if (seg_lo < 0 || seg_lo >= seg_hi) {  // nothing planned for this CTA (uniform over the block)
    record_block_times(p, s_t_start);
    return;
  }

  // TMEM for this CTA (64 of the SM's 512 columns; two CTAs per SM).  The producer does not
  // wait for it: its first requests go out while the MMA warp allocates and the softmax
  // warps build the first q tile.
  uint32_t tmem = 0;
  if (warp != kProducerWarp) {
    if (warp == kMmaWarp) {
      tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), kTmemCols);
      tmem_relinquish();
    }
    tc_fence_before();
    named_barrier_sync(2, (kSoftmaxWarps + 1) * 32);
    tc_fence_after();
    tmem = *tmem_slot;
  }

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    const uint64_t policy = policy_evict_first();
    const int P = p.page_size;
    int fills = 0;  // chunks requested: chunk k goes to K slot k % kKSlots, V slot k % kVSlots
    bool aborted = p.stall_producer != 0;  // failure-path test: send nothing
    for (int s = seg_lo; s < seg_hi && !aborted; ++s) {
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
        int pid[kPieces];
        bool ok = true;
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          const int lp = (c0 + 16 * i) / P;
          pid[i] = __shfl_sync(0xffffffffu, win_val, (lp - win_base) & 31);
          if (16 * i < n) ok = ok && pid[i] >= 0 && pid[i] < p.num_pages;
        }
        // wait until the tensor core has released both slots (S of chunk fills - kKSlots, P.V of
        // chunk fills - kVSlots)
        const int ks = fills % kKSlots, vs = fills % kVSlots;
        bool got = true;
        if (lane == 0) {
          got = mbar_wait_bounded(bar(kBarKEmpty + ks), ((fills / kKSlots) & 1) ^ 1, abort_flag, p.wait_limit_ns) &&
                mbar_wait_bounded(bar(kBarVEmpty + vs), ((fills / kVSlots) & 1) ^ 1, abort_flag, p.wait_limit_ns);
        }
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
          issue_chunk(ks, vs, c0, n, pid, ok, policy);
        }
        __syncwarp();
        ++fills;
      }
    }
    // every slot's last fill must have landed before the CTA may exit (also after an abort:
    // the copies were requested, so they are waited for, within the limit)
    if (lane == 0) {
      for (int k = max(0, fills - kKSlots); k < fills; ++k)
        mbar_wait_drain(bar(kBarKFull + k % kKSlots), (k / kKSlots) & 1, p.wait_limit_ns);
      for (int k = max(0, fills - kVSlots); k < fills; ++k)
        mbar_wait_drain(bar(kBarVFull + k % kVSlots), (k / kVSlots) & 1, p.wait_limit_ns);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // One thread issues every MMA: S of chunk ic as soon as its K tile has landed, the q tile
    // of its segment is written and its score buffer is free; O of chunk ip (ip < is) as
    // soon as the four softmax warps have written its weights.  Chunk k sits in K slot
    // k % kKSlots and V slot k % kVSlots; S, P and O buffers k % 2.  The commit after S hands
    // the K slot back to the producer, the commit after P.V the V slot.
    if (lane == 0) {
      bool aborted = false;
      auto fail = [&](int s) {
        if (!*abort_flag) record_status(hdr_w, DA_DEV_TIMEOUT, s);
        *abort_flag = 1;
        aborted = true;
      };
      // S cursor: segment s_seg (the s_js-th with chunks) holds chunks [.., s_end); segments
      // without chunks are skipped, as on every role
      int s_seg = seg_lo - 1, s_end = 0, s_js = -1;
      bool q_ready = false;
      auto next_segment = [&]() -> bool {
        for (++s_seg; s_seg < seg_hi; ++s_seg) {
          const SegmentInfo si = load_segment(p, segs, s_seg);
          if (!si.valid) continue;
          const int nch = (si.tok1 - si.tok0 + kChunk - 1) / kChunk;
          if (nch == 0) continue;
          s_end += nch;
          ++s_js;
          q_ready = false;
          return true;
        }
        return false;
      };
      bool more = next_segment();  // chunks left whose S is not issued
      int is = 0, ip = 0;
      uint64_t t_last = global_timer_ns();
      for (uint32_t it = 0; !aborted && (more || ip < is); ++it) {
        bool progressed = false;
        // O^T (chunk ip) = V^T . P'^T, first (it hands a V slot back to the producer).  The
        // softmax warps announce the weights after their fold of chunk ip - 2 (the last reader
        // of O buffer ip % 2) and after zeroing the V rows past the loaded tokens, which they
        // do once the V tile has landed.
        const int pvs = ip % kVSlots;
        if (ip < is && mbar_test(bar(kBarPFull + (ip & 1)), (ip >> 1) & 1) &&
            mbar_test(bar(kBarVFull + pvs), (ip / kVSlots) & 1)) {
          tc_fence_after();
          const int pb = ip & 1;
          const uint32_t vt = sbase + kOffV + pvs * kTileBytes;
          const uint32_t pt = sbase + kOffP + pb * 2048;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tc_mma(tmem + 32 + 16 * pb, smem_desc(vt + 4096 * j, 1024, 1024, 2), smem_desc(pt + 512 * j, 128, 128, 0),
                   kIdescPV, j > 0);
          tc_commit(bar(kBarOFull + pb));
          tc_commit(bar(kBarVEmpty + pvs));
          ++ip;
          progressed = true;
        }
        // S^T (chunk ic) = K . Q8^T, with the q tile of the chunk's segment
        if (more && !q_ready) q_ready = mbar_test(bar(kBarQFull + (s_js & 1)), (s_js >> 1) & 1);
        const int ic = is, sb = ic & 1, ks = ic % kKSlots;
        if (more && q_ready && mbar_test(bar(kBarKFull + ks), (ic / kKSlots) & 1) &&
            (ic < 2 || mbar_test(bar(kBarSFree + sb), ((ic >> 1) - 1) & 1))) {
          tc_fence_after();
          const uint32_t kt = sbase + kOffK + ks * kTileBytes;
          const uint32_t q8 = sbase + kOffQ8 + (s_js & 1) * 2048;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tc_mma(tmem + 16 * sb, smem_desc(kt + 32 * j, 16, 1024, 2), smem_desc(q8 + 32 * j, 16, 1024, 2),
                   kIdescS, j > 0);
          tc_commit(bar(kBarSFull + sb));
          tc_commit(bar(kBarKEmpty + ks));
          ++is;
          progressed = true;
          if (is == s_end) more = next_segment();
        }
        if (progressed) {
          t_last = global_timer_ns();
        } else if ((it & 63) == 0 && (*abort_flag || global_timer_ns() - t_last > p.wait_limit_ns)) {
          fail(s_seg);
          break;
        }
      }
      // drain: every MMA this thread issued has completed before TMEM is freed
      tc_commit(bar(kBarDone));
      mbar_wait_timeout(bar(kBarDone), 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int t = threadIdx.x;  // token t of a chunk (S), dim t (O)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    const float score_scale = p.scale_log2 * __ldg(p.k_scale + g);
    const float v_scale = __ldg(p.v_scale + g);
    float* red = reinterpret_cast<float*>(smem + kOffRed);
    float* row_scale = reinterpret_cast<float*>(smem + kOffRowScale);
    const int G = p.group;
    int i = 0, calls = 0;
    auto fail = [&](int s) {
      if (lane == 0) {
        if (!*abort_flag) record_status(hdr_w, DA_DEV_TIMEOUT, s);
        *abort_flag = 1;
      }
    };
    // Every softmax warp takes the same steps (named barriers inside), whatever a wait
    // returns: after a timeout the warps keep walking the plan, skip the tensor-memory
    // reads and write results that the status word marks as invalid.
    auto wait = [&](uint32_t b, uint32_t parity, int s) -> bool {
      const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(b, parity, abort_flag, p.wait_limit_ns));
      if (!ok) fail(s);
      return ok;
    };
    // q of request b as E4M3 rows of q tile jq & 1: row h = hi terms of head h, row 8 + h =
    // lo terms (rows of heads >= G stay 0).  Thread t: head t / 16, dims 8 (t % 16) .. + 7;
    // head h's q is scaled by 2^e_h, e_h putting its largest |q| in [128, 256); 2^-e_h goes
    // into that head's score scale.  Ends with the named barrier and q_full's arrival.
    auto write_q = [&](int b, int jq) {
      const int h = t >> 4, part = t & 15;
      uint2 r0 = make_uint2(0, 0), r1 = make_uint2(0, 0);  // q is 8-byte aligned (API rule)
      if (h < G) {
        const uint2* src =
            reinterpret_cast<const uint2*>(p.q + ((int64_t)b * p.num_q_heads + (int64_t)g * G + h) * kD + 8 * part);
        r0 = __ldg(src);
        r1 = __ldg(src + 1);
      }
      const uint32_t w4[4] = {r0.x, r0.y, r1.x, r1.y};
      float v[8];
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[2 * k] = bf16_lo_to_f32(w4[k]);
        v[2 * k + 1] = bf16_hi_to_f32(w4[k]);
        amax = fmaxf(amax, fmaxf(fabsf(v[2 * k]), fabsf(v[2 * k + 1])));
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const int e = amax > 0.f ? min(max(134 - (int)(__float_as_uint(amax) >> 23), -120), 120) : 0;
      const float up = __uint_as_float((uint32_t)(127 + e) << 23);
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) split_e4m3x2(pack_f16x2(v[2 * k] * up, v[2 * k + 1] * up), hi[k], lo[k]);
      // row r, logical bytes 8 part .. + 7: 16-byte chunk part / 2 (xor r % 8), half part % 2
      uint8_t* tile = smem + kOffQ8 + (jq & 1) * 2048;
      auto q_at = [&](int r) -> uint8_t* { return tile + r * 128 + ((((part >> 1) ^ (r & 7))) << 4) + (part & 1) * 8; };
      *reinterpret_cast<uint2*>(q_at(h)) = make_uint2(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16));
      *reinterpret_cast<uint2*>(q_at(8 + h)) = make_uint2(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16));
      if (part == 0) row_scale[(jq & 1) * 8 + h] = score_scale * __uint_as_float((uint32_t)(127 - e) << 23);
      fence_proxy_async_smem();  // the tensor core reads the q tile
      named_barrier_sync(1, kSoftmaxWarps * 32);
      if (lane == 0) mbar_arrive(bar(kBarQFull + (jq & 1)));
    };
    // the next segment after s that has chunks (its request), or -1
    auto next_with_chunks = [&](int s) -> int {
      for (int s2 = s + 1; s2 < seg_hi; ++s2) {
        const SegmentInfo n2 = load_segment(p, segs, s2);
        if (n2.valid && n2.tok1 > n2.tok0) return n2.b;
      }
      return -1;
    };
    int js = 0;  // segments with chunks seen so far (same count as the MMA thread's)
    for (int s = seg_lo; s < seg_hi; ++s) {
      const SegmentInfo si = load_segment(p, segs, s);
      if (!si.valid) continue;
      const int b = si.b;
      const int nch = (si.tok1 - si.tok0 + kChunk - 1) / kChunk;
      // state, scaled to the reference m_state (per head, base-2 units, P' = 2^(x - m + 8))
      float m_state[8], m_run[8], l_part[8], o_acc[8], f_prev[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        m_state[h] = m_run[h] = -INFINITY;
        l_part[h] = o_acc[h] = 0.f;
        f_prev[h] = 1.f;
      }
      if (nch > 0) {
        // this segment's q tile was written one segment ahead (the first one, now); write the
        // next segment's into the other buffer, whose last user (segment js - 1) is finished
        if (js == 0) write_q(b, 0);
        const int bn = next_with_chunks(s);
        if (bn >= 0) write_q(bn, js + 1);
        const int jcur = js++;
        float rsc[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) rsc[h] = row_scale[(jcur & 1) * 8 + h];

        // fold chunk ic's O^T (its reference reached by factor f from the previous one)
        auto fold = [&](int ic, const float (&f)[8]) {
          const int ob = ic & 1;
          uint32_t o[16];
          if (wait(bar(kBarOFull + ob), (ic >> 1) & 1, s)) {
            tc_fence_after();
            tc_ld16(lane_base + 32 + 16 * ob, o);
            tc_fence_before();
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) o[j] = 0u;
          }
#pragma unroll
          for (int h = 0; h < 8; ++h)
            o_acc[h] = o_acc[h] * f[h] + (__uint_as_float(o[h]) + __uint_as_float(o[8 + h]));
        };
        for (int k = 0; k < nch; ++k, ++i) {
          const int sb = i & 1;
          int n = 0;
          const int vs = i % kVSlots;
          const bool landed = wait(bar(kBarVFull + vs), (i / kVSlots) & 1, s);
          if (landed) n = meta[vs];
          if (landed && t >= n) {  // V rows past the loaded tokens may hold anything (NaN too): zero them
            uint4* vrow = reinterpret_cast<uint4*>(smem + kOffV + vs * kTileBytes + t * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) vrow[c] = make_uint4(0, 0, 0, 0);
          }
          uint32_t sr[16];
          const bool s_ok = wait(bar(kBarSFull + sb), (i >> 1) & 1, s);
          if (s_ok) {
            tc_fence_after();
            tc_ld16(lane_base + 16 * sb, sr);
            tc_fence_before();
          } else {
            n = 0;  // nothing valid: every token masked
#pragma unroll
            for (int j = 0; j < 16; ++j) sr[j] = 0u;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarSFree + sb));
          float x[8], cm[8];
#pragma unroll
          for (int h = 0; h < 8; ++h)
            x[h] = t < n ? (__uint_as_float(sr[h]) + __uint_as_float(sr[8 + h])) * rsc[h] : -INFINITY;
          reduce8<true>(x, cm, red + 32 * (calls++ & 1), warp, lane);
          float f[8], pw[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            m_run[h] = fmaxf(m_run[h], cm[h]);
            const float mi = cm[h] == -INFINITY ? m_state[h] : fmaxf(cm[h], m_run[h] - kFloor);
            const float mu = mi == -INFINITY ? 0.f : mi;
            f[h] = m_state[h] == -INFINITY ? 0.f : fast_exp2(m_state[h] - mu);
            m_state[h] = mi;
            pw[h] = fast_exp2(x[h] - mu + kPShift);  // 0 for masked tokens
            l_part[h] = l_part[h] * f[h] + pw[h];
          }
          uint32_t ph[4], pl[4];
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) split_e4m3x2(pack_f16x2(pw[2 * k2], pw[2 * k2 + 1]), ph[k2], pl[k2]);
          *reinterpret_cast<uint4*>(smem + kOffP + sb * 2048 + 16 * t) =
              make_uint4(ph[0] | (ph[1] << 16), ph[2] | (ph[3] << 16), pl[0] | (pl[1] << 16), pl[2] | (pl[3] << 16));
          fence_proxy_async_smem();  // P' and the zeroed V rows are read by the tensor core
          // this warp's weights of chunk i are in (and its fold of chunk i - 2 is done): the MMA
          // thread issues O^T (chunk i) = V^T . P'^T once all four warps have said so
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarPFull + sb));
          if (k > 0) fold(i - 1, f_prev);
#pragma unroll
          for (int h = 0; h < 8; ++h) f_prev[h] = f[h];
        }
        fold(i - 1, f_prev);
      }

      // ---- the segment's result: per head, O / (sum of weights) and the log-sum-exp
      float lt[8];
      reduce8<false>(l_part, lt, red + 32 * (calls++ & 1), warp, lane);
      // one segment for the request (no load of its segment count): in a dynamic plan, whose
      // segments are never empty, when this one covers all of it; in a static plan, whose
      // requests have S segments each (empty ones too), when S = 1.  With fp32 output the
      // combine writes every request.
      const bool one_segment = p.kind == DA_PLAN_DYNAMIC ? si.tok0 == 0 && si.tok1 == si.len && si.len > 0
                                                         : p.num_ctas == p.batch;
      const bool direct = one_segment && !p.out_f32;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        if (h >= G) break;
        const float val = lt[h] > 0.f ? o_acc[h] * (v_scale / lt[h]) : 0.f;
        const int64_t row = (int64_t)g * G + h;
        if (direct)
          p.out[((int64_t)b * p.num_q_heads + row) * kD + t] = __float2bfloat16_rn(val);
        else
          p.partial_o[((int64_t)s * p.num_q_heads + row) * kD + t] = val;
        if (t == h) {
          const float lse = lt[h] > 0.f ? (m_state[h] + log2f(lt[h]) - kPShift) * 0.69314718055994530942f : -INFINITY;
          if (direct)
            p.lse[(int64_t)b * p.num_q_heads + row] = lse;
          else
            p.partial_lse[(int64_t)s * p.num_q_heads + row] = lse;
        }
      }
    }
  }

  // ---- teardown: every role is done with TMEM
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
  record_block_times(p, s_t_start);
}

}  // namespace

cudaError_t launch_decode_fp8_tc(const DecodeParams& p, const CUtensorMap maps[4], cudaStream_t stream) {
  static_assert(kSmemTc * 2 <= 227 * 1024, "two CTAs per SM must fit");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool configured[64] = {false};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTc);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.num_ctas, (unsigned)p.num_kv_heads, 1);
  cfg.blockDim = dim3(kThreadsTc, 1, 1);
  cfg.dynamicSmemBytes = kSmemTc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel, p, maps[0], maps[1], maps[2], maps[3]);
}

}  // namespace da

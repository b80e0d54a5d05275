// early_start.cuh -- a decode CTA's first segment, derived from seq_lens alone.
//
// The plan (plan.cu) is written by a one-CTA kernel launched just before the decode
// kernel.  Its first segment for CTA c is fixed by the lengths and the plan geometry,
// so a decode CTA can work it out itself and request its first K/V chunks while the
// planner is still running, then check the plan against it once it has landed.  Only
// the launch sequences the library builds itself use this (da_decode_step and the
// one-call steps): there the kernel before the decode is the planner, which writes
// nothing the decode reads except the workspace, so seq_lens, the block table and the
// caches are final when the decode starts.
//
// Formulas (the planner's): n_b = ceil(L_b / T), 0 for a length outside
// [0, max_pages_per_req * page_size]; U = sum_b n_b.
//   dynamic: CTA c owns tiles [floor(cU/C), floor((c+1)U/C)); its first segment is
//            the request b holding tile floor(cU/C), tiles [floor(cU/C) - P_b,
//            min(P_b + n_b, floor((c+1)U/C)) - P_b) with P_b = n_0 + .. + n_{b-1}.
//   static:  CTA c is split s = c mod S of request b = c / S (S = C / B): tiles
//            [min(s k, n_b), min((s+1) k, n_b)) with k = ceil(max_b n_b / S).
#pragma once

#include "da_internal.cuh"

namespace da {

// Largest batch for which the decode kernels derive their first segment themselves
// (every thread walks at most ceil(B / threads) lengths).
constexpr int kEarlyMaxBatch = 1024;

struct FirstSegment {
  int b;             // request, or -1 when the CTA has no tile
  int tile0, tile1;  // tile range relative to the request
};

// Wait (at most limit_ns) for an mbarrier phase whatever the abort flag says: used to let
// the TMA copies a CTA requested land before the CTA exits.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0 && global_timer_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ int tiles_of(const DecodeParams& p, int b) {
  const int L = p.seq_lens[b];
  if (L < 0 || (int64_t)L > p.capacity_tokens) return 0;
  return (int)(((int64_t)L + p.tile_tokens - 1) / p.tile_tokens);
}

// All threads of the block call this (blockDim.x a multiple of 32, at most 1024);
// `scratch` is 72 ints of shared memory.  Contains three __syncthreads.
__device__ inline FirstSegment derive_first_segment(const DecodeParams& p, int cta, int* scratch) {
  const int nt = blockDim.x, t = threadIdx.x, lane = t & 31, warp = t >> 5, nwarps = nt >> 5;
  const int per = (p.batch + nt - 1) / nt;
  const int b0 = min(t * per, p.batch), b1 = min(b0 + per, p.batch);
  int local = 0, lmax = 0;
  for (int b = b0; b < b1; ++b) {
    const int n = tiles_of(p, b);
    local += n;
    lmax = max(lmax, n);
  }
  int incl = local, wmax = lmax;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
    wmax = max(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
  }
  if (lane == 31) scratch[warp] = incl;
  if (lane == 0) scratch[32 + warp] = wmax;
  if (t == 0) scratch[64] = -1;
  __syncthreads();
  int before = 0, U = 0, max_tiles = 0;
  for (int i = 0; i < nwarps; ++i) {
    const int v = scratch[i];
    before += i < warp ? v : 0;
    U += v;
    max_tiles = max(max_tiles, scratch[32 + i]);
  }
  const int excl = before + incl - local;  // tiles of the requests before b0
  if (p.kind == DA_PLAN_DYNAMIC) {
    const int64_t C = p.num_ctas;
    const int64_t u0 = (int64_t)cta * U / C, u1 = (int64_t)(cta + 1) * U / C;
    if (u1 > u0 && excl <= u0 && u0 < (int64_t)excl + local) {  // this thread's requests hold tile u0
      int64_t acc = excl;
      for (int b = b0; b < b1; ++b) {
        const int n = tiles_of(p, b);
        if (u0 < acc + n) {
          scratch[64] = b;
          scratch[65] = (int)(u0 - acc);
          scratch[66] = (int)(min(acc + n, u1) - acc);
          break;
        }
        acc += n;
      }
    }
  } else if (t == 0 && p.batch > 0) {
    const int S = p.num_ctas / p.batch;
    const int b = cta / S, s = cta - b * S;
    const int n = tiles_of(p, b), chunk = (max_tiles + S - 1) / S;
    const int lo = (int)min((int64_t)s * chunk, (int64_t)n), hi = (int)min((int64_t)(s + 1) * chunk, (int64_t)n);
    if (hi > lo) {
      scratch[64] = b;
      scratch[65] = lo;
      scratch[66] = hi;
    }
  }
  __syncthreads();
  FirstSegment fs;
  fs.b = scratch[64];
  fs.tile0 = scratch[65];
  fs.tile1 = scratch[66];
  __syncthreads();  // scratch may be reused
  return fs;
}

}  // namespace da

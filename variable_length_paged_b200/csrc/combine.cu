// combine.cu -- log-sum-exp merge of the per-segment partial results.
//
// A request whose tiles the plan spread over several CTAs has one partial
// (o_i, lse_i) per segment; softmax splits exactly over disjoint token sets,
// so the full result is
//   LSE = M + ln sum_i exp(lse_i - M),   M = max_i lse_i
//   out = sum_i exp(lse_i - LSE) * o_i
// Requests with one segment were written by the decode kernel (with fp32
// output they are merged here too, from their one partial); requests with none
// get out = 0, lse = -inf.
//
// One block per (request, query head); two kernels, chosen by the size of that grid:
//
// combine_kernel (lean, 128 threads, 32 registers): warp w takes segments w, w+4,
// w+8, ... (lse and the lane's head_dim/32 columns loaded together) and keeps its
// own max m_w, sum l_w = sum exp(lse_i - m_w) and accumulator; the four warp states
// are merged in warp order through shared memory.  Sixteen blocks fit on an SM,
// so the grid of a large batch (thousands of blocks, a few segments each) runs in
// one wave.
//
// combine_wide_kernel (256 threads, two passes), for grids of at most
// kWideMaxBlocks blocks, i.e. few requests each split over many segments:
//   1. M = max_i lse_i: the lanes of the eight warps read the lse values side by
//      side (one load per lane covers 256 segments), then one block reduction;
//   2. warp w takes segments w, w+8, w+16, ...: every lane reads the segment's lse
//      (one broadcast load) and its head_dim/32 columns of o_i, eight segments at a
//      time with all loads issued before the arithmetic, and sums
//      l_w = sum exp(lse_i - M) and acc_w = sum exp(lse_i - M) o_i;
//   the eight warp sums are added in warp order.  A request over a few dozen
//   segments costs two load round trips instead of one per four segments.  Its
//   registers (80 a thread) leave room for three blocks per SM, which is why a
//   large grid takes the lean kernel instead.
//
// Both sum in a fixed order, so results are deterministic, and which one runs
// depends only on the batch and head counts.
#include "da_internal.cuh"

namespace da {
namespace {

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const CombineParams p) {
  constexpr int kPer = D / 32;
  constexpr int kWarps = 4;
  __shared__ float4 part[kWarps][32 * kPer / 4];
  __shared__ float ml[kWarps][2];
  grid_dependency_wait();  // partials come from the decode kernel just before
  const int b = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WsLayout WL = ws_layout(p.batch, p.num_ctas, p.max_segments, p.num_kv_heads);
  const int32_t* rsb = p.ws + WL.req_seg_begin;
  const int s0 = rsb[b], s1 = rsb[b + 1];
  const int n = s1 - s0;
  if (n == 1 && !p.out_f32) return;  // written by the decode kernel (uniform over the block)
  const bool ok = s0 >= 0 && s1 <= p.max_segments && n >= 0;
  const int64_t hq = p.num_q_heads;
  const float* plse = p.partial_lse + (int64_t)s0 * hq + h;
  const float* po = p.partial_o + ((int64_t)s0 * hq + h) * D + lane * kPer;

  // this warp's segments, online: m = running max, l = sum exp(lse - m), acc = sum exp(lse - m) o
  float m = -INFINITY, l = 0.f;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  if (ok) {
#pragma unroll 4
    for (int j = warp; j < n; j += kWarps) {
      const float x = __ldcg(plse + (int64_t)j * hq);
      float v[kPer];
      if constexpr (kPer == 4) {
        const float4 t = __ldcg(reinterpret_cast<const float4*>(po + (int64_t)j * hq * D));
        v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
      } else {
        const float2 t = __ldcg(reinterpret_cast<const float2*>(po + (int64_t)j * hq * D));
        v[0] = t.x, v[1] = t.y;
      }
      if (x == -INFINITY) continue;  // an empty partial carries no weight
      const float mn = fmaxf(m, x);
      const float c = expf(m - mn), w = expf(x - mn);  // c = 0 while m is -inf
      l = l * c + w;
#pragma unroll
      for (int k = 0; k < kPer; ++k) acc[k] = acc[k] * c + w * v[k];
      m = mn;
    }
  }
  float* mine = reinterpret_cast<float*>(&part[warp][0]) + lane * kPer;
#pragma unroll
  for (int k = 0; k < kPer; ++k) mine[k] = acc[k];
  if (lane == 0) {
    ml[warp][0] = m;
    ml[warp][1] = l;
  }
  __syncthreads();
  if (warp != 0) return;
  // merge the four warp states in warp order
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, ml[w][0]);
  float L = 0.f, o[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) o[k] = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = expf(ml[w][0] - M);  // 0 for a warp that saw nothing
      L += f * ml[w][1];
      const float* src = reinterpret_cast<const float*>(&part[w][0]) + lane * kPer;
#pragma unroll
      for (int k = 0; k < kPer; ++k) o[k] += f * src[k];
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const float total = L > 0.f ? M + logf(L) : -INFINITY;
  if (p.out_f32) {
    float* dst = reinterpret_cast<float*>(p.out) + ((int64_t)b * hq + h) * D + lane * kPer;
    if constexpr (kPer == 4)
      *reinterpret_cast<float4*>(dst) = make_float4(o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
    else
      *reinterpret_cast<float2*>(dst) = make_float2(o[0] * inv, o[1] * inv);
  } else {
    __nv_bfloat16* dst = p.out + ((int64_t)b * hq + h) * D + lane * kPer;
    if constexpr (kPer == 4) {
      *reinterpret_cast<uint2*>(dst) =
          make_uint2(pack_bf16x2(o[0] * inv, o[1] * inv), pack_bf16x2(o[2] * inv, o[3] * inv));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(o[0] * inv, o[1] * inv);
    }
  }
  if (lane == 0) p.lse[(int64_t)b * hq + h] = total;
}

constexpr int kCombineWarps = 8;

template <int D>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_wide_kernel(const CombineParams p) {
  constexpr int kPer = D / 32;
  constexpr int kU = 8;  // segments per warp with loads in flight together
  __shared__ float4 part[kCombineWarps][32 * kPer / 4];
  __shared__ float red[kCombineWarps][2];
  grid_dependency_wait();  // partials come from the decode kernel just before
  const int b = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WsLayout WL = ws_layout(p.batch, p.num_ctas, p.max_segments, p.num_kv_heads);
  const int32_t* rsb = p.ws + WL.req_seg_begin;
  const int s0 = rsb[b], s1 = rsb[b + 1];
  const int n0 = s1 - s0;
  if (n0 == 1 && !p.out_f32) return;  // written by the decode kernel (uniform over the block)
  const bool ok = s0 >= 0 && s1 <= p.max_segments && n0 >= 0;
  const int n = ok ? n0 : 0;
  const int64_t hq = p.num_q_heads;
  const float* plse = p.partial_lse + (int64_t)s0 * hq + h;
  const float* po = p.partial_o + ((int64_t)s0 * hq + h) * D + lane * kPer;

  // pass 1: M over all segments
  float m = -INFINITY;
  for (int j = threadIdx.x; j < n; j += kCombineWarps * 32) m = fmaxf(m, __ldcg(plse + (int64_t)j * hq));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp][0] = m;
  __syncthreads();
  float M = red[0][0];
#pragma unroll
  for (int w = 1; w < kCombineWarps; ++w) M = fmaxf(M, red[w][0]);

  // pass 2: this warp's share of sum exp(lse_i - M) and sum exp(lse_i - M) o_i
  float l = 0.f, acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  if (M != -INFINITY) {
    for (int j0 = warp; j0 < n; j0 += kCombineWarps * kU) {
      float x[kU], v[kU][kPer];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int j = j0 + kCombineWarps * u;
        x[u] = -INFINITY;
#pragma unroll
        for (int k = 0; k < kPer; ++k) v[u][k] = 0.f;
        if (j < n) {
          x[u] = __ldcg(plse + (int64_t)j * hq);
          if constexpr (kPer == 4) {
            const float4 t = __ldcg(reinterpret_cast<const float4*>(po + (int64_t)j * hq * D));
            v[u][0] = t.x, v[u][1] = t.y, v[u][2] = t.z, v[u][3] = t.w;
          } else {
            const float2 t = __ldcg(reinterpret_cast<const float2*>(po + (int64_t)j * hq * D));
            v[u][0] = t.x, v[u][1] = t.y;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if (x[u] == -INFINITY) continue;  // an empty partial (or none) carries no weight
        const float w = expf(x[u] - M);
        l += w;
#pragma unroll
        for (int k = 0; k < kPer; ++k) acc[k] = fmaf(w, v[u][k], acc[k]);
      }
    }
  }
  float* mine = reinterpret_cast<float*>(&part[warp][0]) + lane * kPer;
#pragma unroll
  for (int k = 0; k < kPer; ++k) mine[k] = acc[k];
  if (lane == 0) red[warp][1] = l;
  __syncthreads();
  if (warp != 0) return;
  // the warp sums, in warp order
  float L = 0.f, o[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) o[k] = 0.f;
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) {
    L += red[w][1];
    const float* src = reinterpret_cast<const float*>(&part[w][0]) + lane * kPer;
#pragma unroll
    for (int k = 0; k < kPer; ++k) o[k] += src[k];
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const float total = L > 0.f ? M + logf(L) : -INFINITY;
  if (p.out_f32) {
    float* dst = reinterpret_cast<float*>(p.out) + ((int64_t)b * hq + h) * D + lane * kPer;
    if constexpr (kPer == 4)
      *reinterpret_cast<float4*>(dst) = make_float4(o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
    else
      *reinterpret_cast<float2*>(dst) = make_float2(o[0] * inv, o[1] * inv);
  } else {
    __nv_bfloat16* dst = p.out + ((int64_t)b * hq + h) * D + lane * kPer;
    if constexpr (kPer == 4) {
      *reinterpret_cast<uint2*>(dst) =
          make_uint2(pack_bf16x2(o[0] * inv, o[1] * inv), pack_bf16x2(o[2] * inv, o[3] * inv));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(o[0] * inv, o[1] * inv);
    }
  }
  if (lane == 0) p.lse[(int64_t)b * hq + h] = total;
}

// Grids up to this many blocks take the wide kernel: one wave of it at three blocks per SM.
constexpr int64_t kWideMaxBlocks = 148 * 3;

template <int D>
cudaError_t launch_combine_d(const CombineParams& p, cudaStream_t stream) {
  const bool wide = (int64_t)p.batch * p.num_q_heads <= kWideMaxBlocks;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.batch, (unsigned)p.num_q_heads, 1);
  cfg.blockDim = dim3(wide ? kCombineWarps * 32 : 128, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return wide ? cudaLaunchKernelEx(&cfg, combine_wide_kernel<D>, p) : cudaLaunchKernelEx(&cfg, combine_kernel<D>, p);
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int head_dim, cudaStream_t stream) {
  if (p.batch == 0) return cudaSuccess;
  if (head_dim == 128) return launch_combine_d<128>(p, stream);
  if (head_dim == 64) return launch_combine_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace da

// combine.cu -- log-sum-exp merge of the per-segment partial results.
//
// A request whose tiles the plan spread over several CTAs has one partial
// (o_i, lse_i) per segment; softmax splits exactly over disjoint token sets,
// so the full result is
//   LSE = M + ln sum_i exp(lse_i - M),   M = max_i lse_i
//   out = sum_i exp(lse_i - LSE) * o_i
// Requests with one segment were written by the decode kernel; requests with
// none get out = 0, lse = -inf.
//
// One 128-thread block per (request, query head).  Every warp reads the
// segments' lse values with its lanes in parallel (max and sum by warp
// reductions, in a fixed order); warp w then accumulates segments w, w+4,
// w+8, ... with each lane owning head_dim/32 columns and the loads unrolled so
// that several are in flight (a request split over many CTAs has tens of
// segments); the four warp sums are added in warp order through shared
// memory.  The order of every sum is fixed, so results are deterministic.
#include "da_internal.cuh"

namespace da {
namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const CombineParams p) {
  constexpr int kPer = D / 32;
  constexpr int kWarps = 4;
  __shared__ float4 part[kWarps - 1][32 * kPer / 4];
  grid_dependency_wait();  // partials come from the decode kernel just before
  const int b = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WsLayout WL = ws_layout(p.batch, p.num_ctas, p.max_segments, p.num_kv_heads);
  const int32_t* rsb = p.ws + WL.req_seg_begin;
  const int s0 = rsb[b], s1 = rsb[b + 1];
  const int n = s1 - s0;
  if (n == 1) return;  // written by the decode kernel (uniform over the block)
  const bool ok = s0 >= 0 && s1 <= p.max_segments && n >= 0;
  const int64_t hq = p.num_q_heads;
  const float* plse = p.partial_lse + (int64_t)s0 * hq + h;

  float M = -INFINITY;
  if (ok)
    for (int i = lane; i < n; i += 32) M = fmaxf(M, __ldcg(plse + i * hq));
  M = warp_max(M);
  float total = -INFINITY;
  if (ok && M != -INFINITY) {
    float sum = 0.f;
    for (int i = lane; i < n; i += 32) sum += expf(__ldcg(plse + i * hq) - M);
    total = M + logf(warp_sum(sum));
  }

  float acc[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) acc[j] = 0.f;
  if (total != -INFINITY) {
    const float* po = p.partial_o + ((int64_t)s0 * hq + h) * D + lane * kPer;
#pragma unroll 8
    for (int j = warp; j < n; j += kWarps) {
      const float wj = expf(__ldcg(plse + j * hq) - total);
      const float* src = po + (int64_t)j * hq * D;
      if constexpr (kPer == 4) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
        acc[0] += wj * v.x;
        acc[1] += wj * v.y;
        acc[2] += wj * v.z;
        acc[3] += wj * v.w;
      } else {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
        acc[0] += wj * v.x;
        acc[1] += wj * v.y;
      }
    }
  }
  // warps 1..3 hand their sums to warp 0, which adds them in warp order
  if (warp > 0) {
    float* dst = reinterpret_cast<float*>(&part[warp - 1][0]) + lane * kPer;
#pragma unroll
    for (int j = 0; j < kPer; ++j) dst[j] = acc[j];
  }
  __syncthreads();
  if (warp != 0) return;
#pragma unroll
  for (int w = 0; w < kWarps - 1; ++w) {
    const float* src = reinterpret_cast<const float*>(&part[w][0]) + lane * kPer;
#pragma unroll
    for (int j = 0; j < kPer; ++j) acc[j] += src[j];
  }
  __nv_bfloat16* dst = p.out + ((int64_t)b * hq + h) * D + lane * kPer;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0], acc[1]);
  }
  if (lane == 0) p.lse[(int64_t)b * hq + h] = total;
}

template <int D>
cudaError_t launch_combine_d(const CombineParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.batch, (unsigned)p.num_q_heads, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel<D>, p);
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int head_dim, cudaStream_t stream) {
  if (p.batch == 0) return cudaSuccess;
  if (head_dim == 128) return launch_combine_d<128>(p, stream);
  if (head_dim == 64) return launch_combine_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace da

// combine.cu -- log-sum-exp merge of the per-segment partial results.
//
// A request whose tiles the plan spread over several CTAs has one partial
// (o_i, lse_i) per segment; softmax splits exactly over disjoint token sets,
// so the full result is
//   LSE = M + ln sum_i exp(lse_i - M),   M = max_i lse_i
//   out = sum_i exp(lse_i - LSE) * o_i
// summed in segment order in fp32.  Requests with one segment were written by
// the decode kernel; requests with none get out = 0, lse = -inf.
//
// One warp per (request, query head); each lane owns head_dim/32 columns.
#include "da_internal.cuh"

namespace da {
namespace {

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const CombineParams p) {
  grid_dependency_wait();  // partials come from the decode kernel just before
  constexpr int kPer = D / 32;
  const int b = blockIdx.x;
  const int h = blockIdx.y * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (h >= p.num_q_heads) return;
  const WsLayout WL = ws_layout(p.batch, p.num_ctas, p.max_segments);
  const int32_t* rsb = p.ws + WL.req_seg_begin;
  const int s0 = rsb[b], s1 = rsb[b + 1];
  const int n = s1 - s0;
  if (n == 1) return;
  __nv_bfloat16* dst = p.out + ((int64_t)b * p.num_q_heads + h) * D + lane * kPer;
  float* lse_dst = p.lse + (int64_t)b * p.num_q_heads + h;
  float acc[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) acc[j] = 0.f;
  float M = -INFINITY;
  const bool ok = s0 >= 0 && s1 <= p.max_segments && n >= 0;
  if (ok) {
    for (int s = s0; s < s1; ++s) M = fmaxf(M, p.partial_lse[(int64_t)s * p.num_q_heads + h]);
  }
  float total = -INFINITY;
  if (ok && M != -INFINITY) {
    float sum = 0.f;
    for (int s = s0; s < s1; ++s) sum += expf(p.partial_lse[(int64_t)s * p.num_q_heads + h] - M);
    total = M + logf(sum);
    for (int s = s0; s < s1; ++s) {
      const float wgt = expf(p.partial_lse[(int64_t)s * p.num_q_heads + h] - total);
      const float* src = p.partial_o + ((int64_t)s * p.num_q_heads + h) * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] += wgt * v.x;
        acc[1] += wgt * v.y;
        acc[2] += wgt * v.z;
        acc[3] += wgt * v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] += wgt * v.x;
        acc[1] += wgt * v.y;
      }
    }
  }
  uint32_t packed[kPer / 2];
#pragma unroll
  for (int j = 0; j < kPer / 2; ++j) packed[j] = pack_bf16x2(acc[2 * j], acc[2 * j + 1]);
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
  } else {
    *reinterpret_cast<uint32_t*>(dst) = packed[0];
  }
  if (lane == 0) *lse_dst = total;
}

template <int D>
cudaError_t launch_combine_d(const CombineParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.batch, (unsigned)((p.num_q_heads + 3) / 4), 1);
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

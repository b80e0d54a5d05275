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
// One 128-thread block per (request, query head), one pass over the partials:
// warp w takes segments w, w+4, w+8, ... (lse and the lane's head_dim/32 columns
// loaded together, unrolled so that several segments are in flight) and keeps
// its own max m_w, sum l_w = sum exp(lse_i - m_w) and accumulator; the four warp
// states are then merged in warp order through shared memory.  Every sum has a
// fixed order, so results are deterministic.
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

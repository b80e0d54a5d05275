// merge.cu -- log-sum-exp merge of results computed over disjoint slices of
// the same requests' caches (one slice per GPU when a long request's KV is
// spread over several GPUs).
//
// "Tencent HPC lands in SGLang, challenging default inference kernels",
// section "Why Tencent HPC matters for online model serving": a longer
// history means more cached data to read; when one request's history is
// split over GPUs, each GPU attends over its slice and the slices combine
// exactly by log-sum-exp, like the split partials inside one GPU:
//   LSE = M + ln sum_j exp(lse_j - M),  out = sum_j exp(lse_j - LSE) out_j.
//
// One warp per output row (request x query x head); lanes own head_dim/32
// columns; parts are summed in part order (fp32), so results are deterministic.
// Parts are bf16 (each GPU's ordinary `out`) or fp32 (steps run with fp32
// output, so that nothing is rounded to bf16 before the merge).
#include "da_internal.cuh"

namespace da {
namespace {

template <int D>
__global__ void __launch_bounds__(128) merge_parts_kernel(const MergeParams p) {
  constexpr int kPer = D / 32;
  grid_dependency_wait();
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  float M = -INFINITY;
  for (int j = 0; j < p.num_parts; ++j) M = fmaxf(M, __ldg(p.part_lse + (int64_t)j * p.rows + row));
  float total = -INFINITY;
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  if (M != -INFINITY) {
    float sum = 0.f;
    for (int j = 0; j < p.num_parts; ++j) sum += expf(__ldg(p.part_lse + (int64_t)j * p.rows + row) - M);
    total = M + logf(sum);
    for (int j = 0; j < p.num_parts; ++j) {
      const float wgt = expf(__ldg(p.part_lse + (int64_t)j * p.rows + row) - total);
      const int64_t at = ((int64_t)j * p.rows + row) * D + lane * kPer;
      float v[kPer];
      if (p.part_out_f32) {
        if constexpr (kPer == 4) {
          const float4 t = __ldg(reinterpret_cast<const float4*>(p.part_out_f32 + at));
          v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
        } else {
          const float2 t = __ldg(reinterpret_cast<const float2*>(p.part_out_f32 + at));
          v[0] = t.x, v[1] = t.y;
        }
      } else if constexpr (kPer == 4) {
        const uint2 t = __ldg(reinterpret_cast<const uint2*>(p.part_out + at));
        v[0] = bf16_lo_to_f32(t.x), v[1] = bf16_hi_to_f32(t.x), v[2] = bf16_lo_to_f32(t.y);
        v[3] = bf16_hi_to_f32(t.y);
      } else {
        const uint32_t t = __ldg(reinterpret_cast<const uint32_t*>(p.part_out + at));
        v[0] = bf16_lo_to_f32(t), v[1] = bf16_hi_to_f32(t);
      }
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] += wgt * v[e];
    }
  }
  __nv_bfloat16* dst = p.out + row * D + lane * kPer;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0], acc[1]);
  }
  if (lane == 0) p.lse[row] = total;
}

template <int D>
cudaError_t launch_merge_d(const MergeParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((p.rows + 3) / 4), 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_parts_kernel<D>, p);
}

}  // namespace

cudaError_t launch_merge(const MergeParams& p, int head_dim, cudaStream_t stream) {
  if (p.rows == 0) return cudaSuccess;
  if (head_dim == 128) return launch_merge_d<128>(p, stream);
  if (head_dim == 64) return launch_merge_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace da

// host_inputs.cuh -- a decode step's inputs brought in from mapped host memory by
// the plan launch itself (one launch instead of a copy per input).
#pragma once

#include "da_internal.cuh"

namespace da {

// n16 16-byte units, then n4 4-byte words, from `src` (the device address of
// mapped, page-locked host memory) to `dst` (device memory).  n16 > 0 needs both
// addresses 16-byte aligned.
struct HostCopy {
  const void* src;
  void* dst;
  int64_t n16;
  int64_t n4;
};

// The plan's block copies the lengths from seq_lens_host (the device address of
// mapped host memory) to seq_lens_dev and plans from that copy; the other blocks
// of the launch run `copies` (block table, q).
struct HostInputs {
  const int32_t* seq_lens_host;
  int32_t* seq_lens_dev;
  HostCopy copies[2];
  int num_copies;
};

cudaError_t launch_plan_host(const PlanParams& p, int kind, const HostInputs& h, cudaStream_t stream);

}  // namespace da

// prepared_step.cuh -- a dynamic decode step (plan, bf16 decode, combine) whose every
// argument check, TMA tensor map and kernel parameter block is done before anything is
// enqueued; launch_prepared_step then only enqueues the three launches.  Used by the
// entry points that run a whole step in one call (defined in api.cu).
#pragma once

#include "da_internal.cuh"

namespace da {

struct PreparedStep {
  PlanParams plan;
  DecodeParams decode;
  CombineParams combine;
  CUtensorMap maps[4];
  da_plan_desc desc;
  int32_t batch, head_dim;
};

// Returns DA_OK or the DA_ERR_* code of the first failing check; enqueues nothing.
int prepare_dynamic_step(const da_problem* prob, const da_plan_desc* desc, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* block_table, const int32_t* seq_lens, void* ws,
                         size_t ws_bytes, float* partial_o, float* partial_lse, void* out, float* lse,
                         PreparedStep* st);

// Enqueues plan, decode and combine on `stream` (a cudaStream_t); DA_ERR_CUDA if a launch is refused.
int launch_prepared_step(const PreparedStep& st, void* stream);

}  // namespace da

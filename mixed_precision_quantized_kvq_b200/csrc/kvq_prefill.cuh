// Launcher of the chunked-prefill attention kernel (kvq_prefill.cu), called
// by the C-ABI layer.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

cudaError_t launch_prefill_attention(const Params& p, const void* q, int q_bf16, const int32_t* cu_q,
                                     const int32_t* lens, int max_q, float sm_scale, float* out, float* lse,
                                     cudaStream_t s);

}  // namespace kvq

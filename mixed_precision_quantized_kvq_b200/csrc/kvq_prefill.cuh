// Launcher of the chunked-prefill attention kernel (kvq_prefill.cu), called
// by the C-ABI layer.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// k_per_channel: key groups run along positions (ring of W + kg - 1 slots).
// one_query: decode (q [B][Hq][d], one query per sequence at its newest
// position, cu_q unused, max_q = 1; empty sequences get out = 0, lse = -inf).
// len_cap: device lengths above it are clamped to it.
cudaError_t launch_prefill_attention(const Params& p, int k_per_channel, int one_query, const void* q,
                                     int q_bf16, const int32_t* cu_q, const int32_t* lens, int len_cap,
                                     int max_q, float sm_scale, float* out, float* lse, cudaStream_t s);

namespace prefill {
struct View;
}
// tensor-core chunked prefill (kvq_prefill_mma.cu): head_dim 128, key groups
// of 32 channels of a token, unrotated keys, value groups dividing 128
bool prefill_mma_supported(const prefill::View& v);
cudaError_t launch_prefill_mma(const prefill::View& v, cudaStream_t s);

}  // namespace kvq

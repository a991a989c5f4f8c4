// Launchers of the per-channel key-group kernels (kvq_channel.cu), called
// by the C-ABI layer for layouts with k_per_channel set.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// Append new tokens: quantize the key groups they complete (keys per
// channel over kg positions, values per token), then write the new
// positions that stay in the window into the ring of W + kg - 1 slots.
cudaError_t launch_append_per_channel(const Params& p, const void* k_new, const void* v_new, int in_bf16,
                                      const int32_t* cu_new, const int32_t* lens, int max_new, cudaStream_t s);

// Reconstruct positions [0, min(len, max_len)) to fp32.
cudaError_t launch_dequantize_per_channel(const Params& p, const int32_t* lens, int max_len, float* k_out,
                                          float* v_out, cudaStream_t s);

}  // namespace kvq

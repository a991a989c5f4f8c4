// Persistent register-fragment decode kernel instantiations for 8-bit keys.
#include "kvq_decode_mma_launch.cuh"

namespace kvq {

cudaError_t launch_decode_mma_k8(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                                 float sl2, float* out, float* lse, float* part, uint32_t* tickets, int ctas, int after_append,
                                 unsigned* status, cudaStream_t s) {
    return mma::launch_kb<8>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, after_append, status, s);
}

}  // namespace kvq

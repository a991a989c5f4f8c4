// Tensor-core decode kernel instantiations for 1-bit keys.
#include "kvq_decode_tc_launch.cuh"

namespace kvq {

cudaError_t launch_decode_tc_k1(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                                float sl2, float* ws_o, float* ws_ml, const DecodePlan& pl, unsigned* status, cudaStream_t s) {
    return tc::launch_kb<1>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, status, s);
}

}  // namespace kvq

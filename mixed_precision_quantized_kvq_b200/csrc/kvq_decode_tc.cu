// Host side of the tensor-core decode kernel (kvq_decode_tc.cuh): which
// layouts it takes, how many CTAs share an SM, and the dispatch over the
// key bit width (the instantiations live in kvq_decode_tc_k{1,2,4,8}.cu so
// they compile in parallel).
#include "kvq_decode_tc.cuh"

namespace kvq {

cudaError_t launch_decode_tc_k1(const Params&, const void*, int, const int32_t*, int, float, float*, float*,
                                const DecodePlan&, unsigned*, cudaStream_t);
cudaError_t launch_decode_tc_k2(const Params&, const void*, int, const int32_t*, int, float, float*, float*,
                                const DecodePlan&, unsigned*, cudaStream_t);
cudaError_t launch_decode_tc_k4(const Params&, const void*, int, const int32_t*, int, float, float*, float*,
                                const DecodePlan&, unsigned*, cudaStream_t);
cudaError_t launch_decode_tc_k8(const Params&, const void*, int, const int32_t*, int, float, float*, float*,
                                const DecodePlan&, unsigned*, cudaStream_t);

static bool bits_ok(int b) { return b == 1 || b == 2 || b == 4 || b == 8; }

bool tc_supported(const Params& p) {
    return p.d == tc::D && p.kg == 32 && p.vg == 128 && p.g >= 1 && p.g <= kMaxGqa && bits_ok(p.kb) &&
           bits_ok(p.vb);
}

// two CTAs per SM when 256 tensor-memory columns and half the shared memory suffice
int tc_ctas_per_sm(const Params& p) {
    return tc::ctas_per_sm(p.kb, p.vb, p.g <= 4 ? 4 : 8);
}

cudaError_t launch_decode_tc(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                             float scale_log2, float* ws_o, float* ws_ml, const DecodePlan& pl, unsigned* status, cudaStream_t s) {
    switch (p.kb) {
        case 1: return launch_decode_tc_k1(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl, status, s);
        case 2: return launch_decode_tc_k2(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl, status, s);
        case 4: return launch_decode_tc_k4(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl, status, s);
        case 8: return launch_decode_tc_k8(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl, status, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace kvq

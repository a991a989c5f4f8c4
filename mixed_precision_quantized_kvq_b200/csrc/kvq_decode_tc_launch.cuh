// Launch of one instantiation of the tensor-core decode kernel; included by
// kvq_decode_tc_k{1,2,4,8}.cu with KVQ_TC_KB set to the key bit width.
#pragma once

#include "kvq_decode_tc.cuh"

namespace kvq {
namespace tc {

template <int KB, int VB, int NHC>
cudaError_t launch_one(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                       float* ws_o, float* ws_ml, const DecodePlan& pl, unsigned* status, cudaStream_t s) {
    using LY = Layout<KB, VB, NHC>;
    auto kern = decode_tc_kernel<KB, VB, NHC>;
    static bool configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::TOTAL);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const dim3 grid(p.hkv, p.batch, pl.grid_x);   // split index outermost
    kern<<<grid, kThreads, LY::TOTAL, s>>>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl.pages_per_split,
                                           pl.window_split, pl.total_splits, status);
    return cudaGetLastError();
}

template <int KB, int VB>
cudaError_t launch_vb(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                      float* ws_o, float* ws_ml, const DecodePlan& pl, unsigned* status, cudaStream_t s) {
    if (p.g <= 4) return launch_one<KB, VB, 4>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, status, s);
    return launch_one<KB, VB, 8>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, status, s);
}

template <int KB>
cudaError_t launch_kb(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                      float* ws_o, float* ws_ml, const DecodePlan& pl, unsigned* status, cudaStream_t s) {
    switch (p.vb) {
        case 1: return launch_vb<KB, 1>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, status, s);
        case 2: return launch_vb<KB, 2>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, status, s);
        case 4: return launch_vb<KB, 4>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, status, s);
        case 8: return launch_vb<KB, 8>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, status, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace tc
}  // namespace kvq

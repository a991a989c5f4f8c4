// Launch of the persistent register-fragment decode kernel
// (kvq_decode_mma.cuh) for one key bit width; included by
// kvq_decode_mma_k{1,2,4,8}.cu with the value bit width and GQA bound
// dispatched here.
#pragma once

#include "kvq_decode_mma.cuh"

namespace kvq {
namespace mma {

// ring slots that fit next to the schedule tables and the query areas
template <int KB, int VB, int NH>
int ring_slots(int batch, int g) {
    using C = Cfg<KB, VB, NH>;
    int r = (kSmemBudget - off_ring<KB, VB, NH>(batch, g)) / C::SLOT;
    if (r > kMaxSlots) r = kMaxSlots;
    // the merge step reuses the ring for one partial per warp
    if (r * C::SLOT < NW * g * PST * int(sizeof(float))) return 0;
    return r >= NW + 2 ? r : 0;
}

template <int KB, int VB, int NH>
cudaError_t launch_one(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                       float* out, float* lse, float* part, uint32_t* tickets, int ctas, unsigned* status, cudaStream_t s) {
    auto kern = decode_mma_kernel<KB, VB, NH>;
    static bool configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const int R = ring_slots<KB, VB, NH>(p.batch, p.g);
    if (R <= 0) return cudaErrorInvalidValue;
    const int bytes = off_ring<KB, VB, NH>(p.batch, p.g) + R * Cfg<KB, VB, NH>::SLOT;
    kern<<<ctas, kThreads, bytes, s>>>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, R, status);
    return cudaGetLastError();
}

template <int KB, int VB>
cudaError_t launch_nh(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                      float* out, float* lse, float* part, uint32_t* tickets, int ctas, unsigned* status, cudaStream_t s) {
    if (p.g <= 4) return launch_one<KB, VB, 4>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, status, s);
    return launch_one<KB, VB, 8>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, status, s);
}

template <int KB>
cudaError_t launch_kb(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                      float* out, float* lse, float* part, uint32_t* tickets, int ctas, unsigned* status, cudaStream_t s) {
    switch (p.vb) {
        case 1: return launch_nh<KB, 1>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, status, s);
        case 2: return launch_nh<KB, 2>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, status, s);
        case 4: return launch_nh<KB, 4>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, status, s);
        case 8: return launch_nh<KB, 8>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, status, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace mma
}  // namespace kvq

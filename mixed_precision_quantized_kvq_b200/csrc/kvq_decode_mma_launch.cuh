// Launch of the persistent register-fragment decode kernel
// (kvq_decode_mma.cuh) for one key bit width; included by
// kvq_decode_mma_k{1,2,4,8}.cu with the value bit width and GQA bound
// dispatched here.
#pragma once

#include <cudaTypedefs.h>

#include "kvq_decode_mma.cuh"

namespace kvq {
namespace mma {

// Tensor maps of the bf16 window rings [batch * Hkv * W rows][128 channels]:
// boxes of 16 rows x 64 channels with the 128-byte swizzle.  The encoder is
// the driver's cuTensorMapEncodeTiled, looked up through the runtime.
inline cudaError_t window_maps(const Params& p, CUtensorMap* mk, CUtensorMap* mv) {
    memset(mk, 0, sizeof(*mk));
    memset(mv, 0, sizeof(*mv));
    if (p.W <= 0 || !p.k_win || !p.v_win) return cudaSuccess;     // no window units are issued
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(p.batch) * p.hkv * p.W};
    const cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    const cuuint32_t box[2] = {64, 16}, estr[2] = {1, 1};
    for (int i = 0; i < 2; ++i) {
        const CUresult r = encode(i ? mv : mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, i ? (void*)p.v_win : (void*)p.k_win,
                                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    return cudaSuccess;
}

// ring slots that fit next to the schedule tables and the query areas
// ring slots per warp that fit beside the schedule tables and the per-warp
// areas (0: the layout does not fit this kernel)
template <int KB, int VB, int NH>
int ring_slots(int batch, int g) {
    using C = Cfg<KB, VB, NH>;
    int r = (kSmemBudget - 1024 - off_ring<KB, VB, NH>(batch, g)) / (C::NW * C::SLOT);   // 1024: ring alignment
    if (r > kMaxSpw) r = kMaxSpw;
    // the merge step reuses the ring for one partial per warp
    if (r * C::NW * C::SLOT < C::NW * g * PST * int(sizeof(float))) return 0;
    return r >= 2 ? r : 0;
}

template <int KB, int VB, int NH>
cudaError_t launch_one(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                       float* out, float* lse, float* part, uint32_t* tickets, int ctas, int after_append, unsigned* status, cudaStream_t s) {
    auto kern = decode_mma_kernel<KB, VB, NH>;
    static bool configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    using C = Cfg<KB, VB, NH>;
    const int spw = ring_slots<KB, VB, NH>(p.batch, p.g);
    if (spw <= 0) return cudaErrorInvalidValue;
    const int bytes = off_ring<KB, VB, NH>(p.batch, p.g) + 1024 + spw * C::NW * C::SLOT;
    CUtensorMap mk, mv;
    const cudaError_t em = window_maps(p, &mk, &mv);
    if (em != cudaSuccess) return em;
    // no CTA waits for another (pairs split between CTAs are merged by the CTA
    // that finishes last), so a plain launch of one CTA per SM; right after an
    // append, as its programmatic dependent (the kernel waits for the append's
    // results before it reads the cache)
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(C::NW * 32);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = after_append ? attr : nullptr;
    cfg.numAttrs = after_append ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, spw,
                              after_append, status, mk, mv);
}

template <int KB, int VB>
cudaError_t launch_nh(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                      float* out, float* lse, float* part, uint32_t* tickets, int ctas, int after_append, unsigned* status, cudaStream_t s) {
    if (p.g <= 4) return launch_one<KB, VB, 4>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, after_append, status, s);
    return launch_one<KB, VB, 8>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, after_append, status, s);
}

template <int KB>
cudaError_t launch_kb(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                      float* out, float* lse, float* part, uint32_t* tickets, int ctas, int after_append, unsigned* status, cudaStream_t s) {
    switch (p.vb) {
        case 1: return launch_nh<KB, 1>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, after_append, status, s);
        case 2: return launch_nh<KB, 2>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, after_append, status, s);
        case 4: return launch_nh<KB, 4>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, after_append, status, s);
        case 8: return launch_nh<KB, 8>(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, ctas, after_append, status, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace mma
}  // namespace kvq

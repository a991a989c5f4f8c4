// Internal declarations of the kvq CUDA library (sm_100a).
// Kernel parameter block, cache addressing and the launchers that the C-ABI
// layer (kvq_api.cu) calls.  Nothing here is visible outside the library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kPage = 64;          // tokens per page
constexpr int kMaxGqa = 8;         // query heads per kv-head
constexpr int kTcWindowPerCta = 64; // window positions per window CTA of the tensor-core decode

// Flat copy of kvq_layout + kvq_cache with the derived strides kernels use.
struct Params {
    int d, hq, hkv, g;             // head_dim, heads, gqa ratio
    int kb, vb, kg, vg;            // bits and group sizes
    int nkg, nvg;                  // groups per row
    int W;                         // window
    int rotate;
    const int8_t* signs;
    uint8_t* k_codes;
    uint8_t* v_codes;
    uint32_t* k_meta;              // {u16 scale, u16 zero} per group
    uint32_t* v_meta;
    __nv_bfloat16* k_win;
    __nv_bfloat16* v_win;
    const int32_t* page_table;
    int batch, max_pages, num_pages;
    int krow_bytes;                // d*kb/8
    int vchan_bytes;               // page*vb/8
    int kch, vch;                  // chunk bytes: min(16, row bytes)
};

// ---- cache addressing (layout documented in kvq.h) ----------------------
// Code rows longer than 16 bytes are stored as 16-byte chunks, chunk-major
// inside the (page, kv-head) block, so that one thread per token (keys) or
// per channel (values) reading chunk i hits consecutive 16-byte units.
__device__ __forceinline__ uint8_t* k_block(const Params& p, int page, int h) {
    return p.k_codes + (size_t(page) * p.hkv + h) * size_t(kPage) * p.krow_bytes;
}
__device__ __forceinline__ uint32_t* k_word(const Params& p, int page, int h, int slot, int w) {
    const int byte = 4 * w;
    return reinterpret_cast<uint32_t*>(k_block(p, page, h) + (byte / p.kch) * (kPage * p.kch) + slot * p.kch +
                                       (byte % p.kch));
}
__device__ __forceinline__ uint32_t* k_meta_row(const Params& p, int page, int h, int slot) {
    return p.k_meta + ((size_t(page) * p.hkv + h) * kPage + slot) * p.nkg;
}
__device__ __forceinline__ uint8_t* v_block(const Params& p, int page, int h) {
    return p.v_codes + (size_t(page) * p.hkv + h) * size_t(p.d) * p.vchan_bytes;
}
__device__ __forceinline__ uint32_t* v_word(const Params& p, int page, int h, int j, int w) {
    const int byte = 4 * w;
    return reinterpret_cast<uint32_t*>(v_block(p, page, h) + (byte / p.vch) * (p.d * p.vch) + j * p.vch +
                                       (byte % p.vch));
}
__device__ __forceinline__ uint32_t* v_meta_row(const Params& p, int page, int h, int slot) {
    return p.v_meta + ((size_t(page) * p.hkv + h) * kPage + slot) * p.nvg;
}
__device__ __forceinline__ size_t win_off(const Params& p, int b, int h, int pos) {
    return ((size_t(b) * p.hkv + h) * p.W + (pos % p.W)) * p.d;
}
// physical page of logical page `lp` of sequence b, or -1 when absent
__device__ __forceinline__ int phys_page(const Params& p, int b, int lp) {
    if (lp < 0 || lp >= p.max_pages) return -1;
    int pg = __ldg(p.page_table + size_t(b) * p.max_pages + lp);
    return (pg >= 0 && pg < p.num_pages) ? pg : -1;
}

// meta word -> (scale, zero) as fp32
__device__ __forceinline__ float2 meta_f2(uint32_t w) {
    __half2 h = *reinterpret_cast<const __half2*>(&w);
    return __half22float2(h);   // .x = scale, .y = zero
}

// ---- key-only rotation (Walsh-Hadamard), shared by append and decode ----
template <int D>
struct RotScale;
template <>
struct RotScale<64> { static constexpr float v = 0.125f; };
template <>
struct RotScale<128> { static constexpr float v = 0.0883883476483184405f; };  // 1/sqrt(128)

// x holds channels lane*CPL .. lane*CPL+CPL-1.  Sylvester-ordered transform:
// butterflies (a, b) -> (a + b, a - b) over strides 1, 2, ..., D/2.
template <int D>
__device__ __forceinline__ void rotate_warp(float (&x)[D / 32], const int8_t* signs, int lane) {
    constexpr int CPL = D / 32;
#pragma unroll
    for (int i = 0; i < CPL; ++i) x[i] = __fmul_rn(x[i], (float)__ldg(signs + lane * CPL + i));
#pragma unroll
    for (int s = 1; s < CPL; s <<= 1) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            if (!(i & s)) {
                float a = x[i], b = x[i + s];
                x[i] = __fadd_rn(a, b);
                x[i + s] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            float o = __shfl_xor_sync(0xffffffffu, x[i], m);
            x[i] = (lane & m) ? __fsub_rn(o, x[i]) : __fadd_rn(x[i], o);
        }
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i) x[i] = __fmul_rn(x[i], RotScale<D>::v);
}

// ---- launchers -----------------------------------------------------------
struct DecodePlan {
    int mma;            // 1: persistent register-fragment tensor-core kernel (no combine launch)
    int ctas;           // its grid: one CTA per SM at most
    int after_append;   // 1: launched right after a one-launch append on the same stream, as its
                        //    programmatic dependent (start-up overlaps the append)
    int tc;             // 1: two-phase tcgen05 kernel, 0: CUDA-core kernel (when mma == 0)
    int splits_q;       // splits over quantized pages
    int pages_per_split;
    int window_split;   // partial slots of the bf16 window (CUDA-core kernel: 0 or 1; tensor-core
                        // kernel: window CTAs per (sequence, kv-head), in slots 0 .. window_split-1)
    int total_splits;   // partial slots per (sequence, query head)
    int grid_x;         // CTAs per (sequence, kv-head)
    int window_slot;    // slot index of the window partial
};
// persistent register-fragment tensor-core decode (kvq_decode_mma.cuh), one key bit width per file
cudaError_t launch_decode_mma_k1(const Params&, const void*, int, const int32_t*, int, float, float*, float*, float*,
                                 uint32_t*, int, int, unsigned*, cudaStream_t);
cudaError_t launch_decode_mma_k2(const Params&, const void*, int, const int32_t*, int, float, float*, float*, float*,
                                 uint32_t*, int, int, unsigned*, cudaStream_t);
cudaError_t launch_decode_mma_k4(const Params&, const void*, int, const int32_t*, int, float, float*, float*, float*,
                                 uint32_t*, int, int, unsigned*, cudaStream_t);
cudaError_t launch_decode_mma_k8(const Params&, const void*, int, const int32_t*, int, float, float*, float*, float*,
                                 uint32_t*, int, int, unsigned*, cudaStream_t);
// decode path selection: 0 = automatic, 1 = CUDA cores, 2 = tensor cores
extern int g_decode_path;
DecodePlan plan_decode(const Params& p, int batch, int max_len, int sm_count);
bool tc_supported(const Params& p);
bool mma_supported(const Params& p, int batch);
// workspace of the persistent kernel: merge partials of `ctas` CTAs, then one
// ticket per (sequence, kv-head); returns the bytes, and the tickets' offset
size_t mma_workspace_layout(const Params& p, int batch, int ctas, size_t* off_tickets);
int tc_ctas_per_sm(const Params& p);
cudaError_t launch_decode_tc(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                             float scale_log2, float* ws_o, float* ws_ml, const DecodePlan& pl, unsigned* status,
                             cudaStream_t s);
size_t decode_workspace_bytes(const Params& p, int batch, const DecodePlan& plan);

// decode for key groups along positions (kvq_decode_pc.cu): head_dim 128, up
// to 8 query heads per kv-head, key groups of 16/32/64 positions, unrotated
bool decode_pc_supported(const Params& p, int max_len);
// CTAs per (sequence, kv-head) of the per-channel decode: more than one only
// when the pairs leave SMs without a CTA (all CTAs in one wave), at most 8,
// and at least eight 64-position tiles per CTA at max_len
int pc_splits(const Params& p, int batch, int max_len, int sms);
// workspace of a split per-channel decode: partials [pairs][splits][8 heads][132]
// floats, then one merge ticket per pair (zero-filled once)
size_t pc_workspace_bytes(const Params& p, int batch, int splits);
cudaError_t launch_decode_per_channel(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                                      float sm_scale, float* out, float* lse, void* ws, int splits, cudaStream_t s);
// the append of max_new tokens per sequence is one launch of the small-append
// kernel (which lets a programmatic dependent start early)
bool append_is_one_launch(const Params& p, int max_new);
cudaError_t launch_quantize_append(const Params& p, const void* k_new, const void* v_new,
                                   int in_bf16, const int32_t* cu_new, const int32_t* lens,
                                   int max_new, cudaStream_t s);
cudaError_t launch_dequantize(const Params& p, const int32_t* lens, int max_len, float* k_out,
                              float* v_out, cudaStream_t s);
cudaError_t launch_rotate_keys(const Params& p, const void* k, int in_bf16, int rows, float* out,
                               cudaStream_t s);
cudaError_t launch_decode(const Params& p, const void* q, int q_bf16, const int32_t* lens,
                          int max_len, float sm_scale, float* out, float* lse, void* ws,
                          const DecodePlan& plan, cudaStream_t s);
// decode diagnostics (device words the decode kernels count into): [0] bounded
// waits that expired, [1] tickets found above their count.  Read and
// optionally cleared by decode_status (blocking).
cudaError_t decode_status(unsigned* wait_timeouts, unsigned* bad_tickets, bool clear);

}  // namespace kvq

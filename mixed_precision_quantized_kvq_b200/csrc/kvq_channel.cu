// Per-channel key groups: CUDA kernels around the CTA bodies in
// kvq_channel_body.cuh, and their launchers.
//
// Append = two launches on the caller's stream: the group kernel
// (grid: groups completed by the longest append x kv-heads x sequences,
// 512 threads, about kg*d*10 bytes of shared memory) reads ring slots of the
// positions it quantizes; the ring kernel (grid: kv-heads x sequences)
// then writes the new positions that stay in the window.
#include "kvq_channel.cuh"
#include "kvq_channel_body.cuh"

namespace kvq {
namespace {

struct ChanCtx {
    float* s;
    __device__ int tid() const { return threadIdx.x; }
    __device__ int nthreads() const { return blockDim.x; }
    __device__ int bx() const { return blockIdx.x; }
    __device__ int by() const { return blockIdx.y; }
    __device__ int bz() const { return blockIdx.z; }
    __device__ float* smem() const { return s; }
    __device__ void sync() const { __syncthreads(); }
    __device__ uint16_t f2h_rd(float x) const { return __half_as_ushort(__float2half_rd(x)); }
    __device__ uint16_t f2h_ru(float x) const { return __half_as_ushort(__float2half_ru(x)); }
    __device__ float sub_ru(float a, float b) const { return __fsub_ru(a, b); }
    __device__ float div_ru(float a, float b) const { return __fdiv_ru(a, b); }
    __device__ float sub_rn(float a, float b) const { return __fsub_rn(a, b); }
    __device__ float div_rn(float a, float b) const { return __fdiv_rn(a, b); }
    __device__ float mul_rn(float a, float b) const { return __fmul_rn(a, b); }
    __device__ uint16_t f2bf_rn(float x) const { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
    __device__ void atomic_and(uint32_t* p, uint32_t v) const { atomicAnd(p, v); }
    __device__ void atomic_or(uint32_t* p, uint32_t v) const { atomicOr(p, v); }
};

__global__ void __launch_bounds__(chan::kGroupThreads) append_groups_kernel(chan::View v) {
    extern __shared__ __align__(16) float smem[];
    ChanCtx cx{smem};
    chan::append_groups_body(cx, v);
}

__global__ void __launch_bounds__(chan::kThreads) ring_write_kernel(chan::View v) {
    ChanCtx cx{nullptr};
    chan::ring_write_body(cx, v);
}

__global__ void __launch_bounds__(chan::kThreads) dequant_pc_kernel(chan::View v) {
    ChanCtx cx{nullptr};
    chan::dequant_body(cx, v);
}

chan::View make_view(const Params& p) {
    chan::View v{};
    v.d = p.d;
    v.hkv = p.hkv;
    v.kb = p.kb;
    v.vb = p.vb;
    v.kg = p.kg;
    v.vg = p.vg;
    v.nvg = p.nvg;
    v.W = p.W;
    v.R = p.W + p.kg - 1;
    v.k_codes = p.k_codes;
    v.v_codes = p.v_codes;
    v.k_meta = p.k_meta;
    v.v_meta = p.v_meta;
    v.k_win = reinterpret_cast<uint16_t*>(p.k_win);
    v.v_win = reinterpret_cast<uint16_t*>(p.v_win);
    v.page_table = p.page_table;
    v.batch = p.batch;
    v.max_pages = p.max_pages;
    v.num_pages = p.num_pages;
    v.kchan_bytes = chan::kPage * p.kb / 8;
    v.vchan_bytes = chan::kPage * p.vb / 8;
    v.kch = v.kchan_bytes < 16 ? v.kchan_bytes : 16;
    v.vch = v.vchan_bytes < 16 ? v.vchan_bytes : 16;
    return v;
}

}  // namespace

cudaError_t launch_append_per_channel(const Params& p, const void* k_new, const void* v_new, int in_bf16,
                                      const int32_t* cu_new, const int32_t* lens, int max_new, cudaStream_t s) {
    chan::View v = make_view(p);
    v.k_new = k_new;
    v.v_new = v_new;
    v.in_bf16 = in_bf16;
    v.cu_new = cu_new;
    v.lens = lens;
    // opt in once per device, for the largest size (d 128, groups of 64)
    static bool configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    cudaError_t e;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(append_groups_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(chan::append_smem_bytes(128, 64, 8)));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const size_t sm = chan::append_smem_bytes(p.d, p.kg, p.nvg);
    const int groups = (max_new + p.kg - 1) / p.kg;
    append_groups_kernel<<<dim3(groups, p.hkv, p.batch), chan::kGroupThreads, sm, s>>>(v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ring_write_kernel<<<dim3(p.hkv, p.batch), chan::kThreads, 0, s>>>(v);
    return cudaGetLastError();
}

cudaError_t launch_dequantize_per_channel(const Params& p, const int32_t* lens, int max_len, float* k_out,
                                          float* v_out, cudaStream_t s) {
    chan::View v = make_view(p);
    v.lens = lens;
    v.max_len = max_len;
    v.k_out = k_out;
    v.v_out = v_out;
    dequant_pc_kernel<<<dim3((max_len + chan::kPage - 1) / chan::kPage, p.hkv, p.batch), chan::kThreads, 0, s>>>(v);
    return cudaGetLastError();
}

}  // namespace kvq

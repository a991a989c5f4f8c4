// Chunked-prefill attention over the quantized cache: the CUDA kernel around
// the per-CTA body in kvq_prefill_body.cuh, and its launcher.
//
// Grid: (query tiles of the longest chunk, kv-heads, sequences); 256 threads
// and about 117 KB (150 KB with key rotation) of dynamic shared memory per
// CTA at head_dim 128.  CTAs whose query tile lies past their sequence's
// chunk return at once.
#include "kvq_prefill.cuh"
#include "kvq_prefill_body.cuh"

namespace kvq {
namespace {

struct DevCtx {
    float* s;
    __device__ int tid() const { return threadIdx.x; }
    __device__ int bx() const { return blockIdx.x; }
    __device__ int by() const { return blockIdx.y; }
    __device__ int bz() const { return blockIdx.z; }
    __device__ float* smem() const { return s; }
    __device__ void sync() const { __syncthreads(); }
    __device__ float warp_max(float x) const {
#pragma unroll
        for (int m = 16; m; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
        return x;
    }
    __device__ float warp_sum(float x) const {
#pragma unroll
        for (int m = 16; m; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
        return x;
    }
};

template <int D>
__global__ void __launch_bounds__(prefill::kThreads) prefill_attention_kernel(prefill::View v) {
    extern __shared__ __align__(16) float smem[];
    DevCtx cx{smem};
    prefill::body<D>(cx, v);
}

template <int D>
cudaError_t launch_d(const prefill::View& v, cudaStream_t s) {
    // opt in once per device, for the largest size (with rotation)
    static bool configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(prefill_attention_kernel<D>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   int(prefill::smem_bytes(D, 1)));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const size_t sm = prefill::smem_bytes(D, v.rotate);
    const int qpc = prefill::queries_per_cta(v.g);
    dim3 grid((v.max_q + qpc - 1) / qpc, v.hkv, v.batch);
    prefill_attention_kernel<D><<<grid, prefill::kThreads, sm, s>>>(v);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attention(const Params& p, int k_per_channel, int one_query, const void* q,
                                     int q_bf16, const int32_t* cu_q, const int32_t* lens, int len_cap,
                                     int max_q, float sm_scale, float* out, float* lse, cudaStream_t s) {
    prefill::View v{};
    v.d = p.d;
    v.hq = p.hq;
    v.hkv = p.hkv;
    v.g = p.g;
    v.kb = p.kb;
    v.vb = p.vb;
    v.kg = p.kg;
    v.vg = p.vg;
    v.nkg = p.nkg;
    v.nvg = p.nvg;
    v.W = p.W;
    v.rotate = p.rotate;
    v.kpc = k_per_channel;
    v.R = k_per_channel ? p.W + p.kg - 1 : p.W;
    v.kchan_bytes = prefill::kTile * p.kb / 8;
    v.kchc = v.kchan_bytes < 16 ? v.kchan_bytes : 16;
    v.one_query = one_query;
    v.signs = p.signs;
    v.k_codes = p.k_codes;
    v.v_codes = p.v_codes;
    v.k_meta = p.k_meta;
    v.v_meta = p.v_meta;
    v.k_win = reinterpret_cast<const uint16_t*>(p.k_win);
    v.v_win = reinterpret_cast<const uint16_t*>(p.v_win);
    v.page_table = p.page_table;
    v.batch = p.batch;
    v.max_pages = p.max_pages;
    v.num_pages = p.num_pages;
    v.krow_bytes = p.krow_bytes;
    v.vchan_bytes = p.vchan_bytes;
    v.kch = p.kch;
    v.vch = p.vch;
    v.q = q;
    v.q_bf16 = q_bf16;
    v.cu_q = cu_q;
    v.lens = lens;
    v.len_cap = len_cap;
    v.max_q = max_q;
    v.scale_log2 = sm_scale * 1.4426950408889634f;
    v.out = out;
    v.lse = lse;
    if (prefill_mma_supported(v)) return launch_prefill_mma(v, s);
    return p.d == 128 ? launch_d<128>(v, s) : launch_d<64>(v, s);
}

}  // namespace kvq

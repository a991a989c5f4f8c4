// Quantize / append, window ring, key rotation and reconstruction kernels.
//
// Group quantizer ("Kuantisasi KV cache mengganggu attention ...", section
// "Granularitas kuantisasi menentukan nilai yang berbagi scale"): per token
// and group of contiguous channels, fp32 min/max by warp shuffles, then
//   zero  = fp16 round-down(min)
//   scale = fp16 round-up( (max - zero) /ru (2^b - 1) )  (fp32 steps rounded up)
//   code  = clamp(rint((x - zero) / scale), 0, 2^b - 1)   (IEEE fp32, RN)
// Every fp32 step is a single intrinsic with an explicit rounding mode, so
// the result does not depend on contraction or fast-math.
//
// Recent-token window ("Pertumbuhan cache mengubah trade pada serving"):
// the newest W positions live in a bf16 ring; a position is quantized when
// it leaves the ring.  Key-only rotation ("Quantize What Counts ...",
// Resultaten): keys are multiplied by diag(signs) * H / sqrt(d) (fast
// Walsh-Hadamard transform across the warp) before quantization.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr unsigned FULL = 0xffffffffu;

// Quantize the warp's row (lane holds CPL contiguous channels) in groups of
// `group` channels at `bits`.  Returns codes in c[], and (scale, zero) of the
// lane's group as fp16 bit patterns packed {scale | zero << 16}.
template <int D>
__device__ __forceinline__ uint32_t quantize_warp(const float (&x)[D / 32], int group, int bits,
                                                  uint32_t (&c)[D / 32]) {
    constexpr int CPL = D / 32;
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int i = 1; i < CPL; ++i) {
        mn = fminf(mn, x[i]);
        mx = fmaxf(mx, x[i]);
    }
    const int lanes = group / CPL;   // lanes sharing one group (power of two)
    for (int o = 1; o < lanes; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
    }
    if (mn == 0.0f) mn = 0.0f;       // canonical +0
    if (mx == 0.0f) mx = 0.0f;
    const float qmax = (float)((1 << bits) - 1);
    const __half zh = __float2half_rd(mn);
    const float zf = __half2float(zh);
    const float r = __fsub_ru(mx, zf);
    const float s32 = __fdiv_ru(r, qmax);
    __half sh = __float2half_ru(s32);
    const float sf = __half2float(sh);
    if (sf == 0.0f) sh = __ushort_as_half(0);
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        float code = 0.0f;
        if (sf != 0.0f) {
            float t = __fdiv_rn(__fsub_rn(x[i], zf), sf);
            code = fminf(fmaxf(rintf(t), 0.0f), qmax);
        }
        c[i] = (uint32_t)code;
    }
    return (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
}

template <int D>
__device__ __forceinline__ void load_row(const void* src, int in_bf16, size_t off, int lane,
                                         float (&x)[D / 32]) {
    constexpr int CPL = D / 32;
    if (in_bf16) {
        const __nv_bfloat16* s = reinterpret_cast<const __nv_bfloat16*>(src) + off + lane * CPL;
#pragma unroll
        for (int i = 0; i < CPL; ++i) x[i] = __bfloat162float(s[i]);
    } else {
        const float* s = reinterpret_cast<const float*>(src) + off + lane * CPL;
#pragma unroll
        for (int i = 0; i < CPL; ++i) x[i] = s[i];
    }
}

// One CTA quantizes a 32-aligned block of positions of one (sequence,
// kv-head): warps take 8 positions each; key rows and metadata are written
// per position; value codes (stored per channel, 32/vb tokens per word) are
// staged in shared memory and written as whole words once the block is done.
// Words that also hold positions outside [q0, q1) keep those bits.
template <int D>
__global__ void __launch_bounds__(128) quantize_pages_kernel(Params p, const void* __restrict__ k_new,
                                                             const void* __restrict__ v_new, int in_bf16,
                                                             const int32_t* __restrict__ cu_new,
                                                             const int32_t* __restrict__ lens) {
    constexpr int CPL = D / 32;
    __shared__ uint8_t vstage[D][32];
    const int b = blockIdx.z, h = blockIdx.y;
    const int L = lens[b];
    const int n = cu_new[b + 1] - cu_new[b];
    const int q0 = max(0, L - p.W), q1 = max(0, L + n - p.W);
    const int base = (q0 & ~31) + 32 * blockIdx.x;
    if (base >= q1 || n < 0 || L < 0) return;
    const int lp = base / kPage;
    const int page = phys_page(p, b, lp);
    if (page < 0) return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    for (int k = 0; k < 8; ++k) {
        const int slot32 = warp * 8 + k;
        const int pos = base + slot32;
        if (pos < q0 || pos >= q1) continue;            // warp-uniform
        float kx[CPL], vx[CPL];
        if (pos < L) {                                   // leaving the window ring
            size_t off = win_off(p, b, h, pos);
            load_row<D>(p.k_win, 1, off, lane, kx);
            load_row<D>(p.v_win, 1, off, lane, vx);
        } else {
            size_t off = (size_t(cu_new[b] + pos - L) * p.hkv + h) * D;
            load_row<D>(k_new, in_bf16, off, lane, kx);
            load_row<D>(v_new, in_bf16, off, lane, vx);
        }
        if (p.rotate) rotate_warp<D>(kx, p.signs, lane);
        const int slot = pos % kPage;
        // ---- keys: token row
        uint32_t kc[CPL];
        uint32_t km = quantize_warp<D>(kx, p.kg, p.kb, kc);
        if ((lane * CPL) % p.kg == 0) k_meta_row(p, page, h, slot)[(lane * CPL) / p.kg] = km;
        uint32_t bitsv = 0;
#pragma unroll
        for (int i = 0; i < CPL; ++i) bitsv |= kc[i] << (p.kb * i);
        const int lane_bits = CPL * p.kb;                // <= 32
        const int lpw = 32 / lane_bits;                  // lanes per 32-bit word
        bitsv <<= (lane % lpw) * lane_bits;
        for (int o = 1; o < lpw; o <<= 1) bitsv |= __shfl_xor_sync(FULL, bitsv, o);
        if (lane % lpw == 0) *k_word(p, page, h, slot, lane / lpw) = bitsv;
        // ---- values: metadata per token, codes staged per channel
        uint32_t vc[CPL];
        uint32_t vm = quantize_warp<D>(vx, p.vg, p.vb, vc);
        if ((lane * CPL) % p.vg == 0) v_meta_row(p, page, h, slot)[(lane * CPL) / p.vg] = vm;
#pragma unroll
        for (int i = 0; i < CPL; ++i) vstage[lane * CPL + i][slot32] = (uint8_t)vc[i];
    }
    __syncthreads();
    // value words: channel j, word wi covers 32/vb consecutive slots
    const int per = 32 / p.vb;                           // slots per word
    const int words = 32 / per;                          // words in this 32-slot block
    const int slot0 = base % kPage;
    for (int t = threadIdx.x; t < D * words; t += blockDim.x) {
        const int j = t / words, wi = t % words;
        uint32_t* dst = v_word(p, page, h, j, (slot0 + wi * per) / per);
        uint32_t word = 0, keep = 0;
        const uint32_t fmask = (1u << p.vb) - 1u;
        for (int i = 0; i < per; ++i) {
            const int s32 = wi * per + i;
            const int pos = base + s32;
            if (pos >= q0 && pos < q1) word |= ((uint32_t)vstage[j][s32] & fmask) << (p.vb * i);
            else keep |= fmask << (p.vb * i);
        }
        if (keep) word |= *dst & keep;
        *dst = word;
    }
}

// Newest positions [max(L, L+n-W), L+n) into the bf16 ring; one warp per
// position and kv-head.
template <int D>
__global__ void __launch_bounds__(128) window_write_kernel(Params p, const void* __restrict__ k_new,
                                                           const void* __restrict__ v_new, int in_bf16,
                                                           const int32_t* __restrict__ cu_new,
                                                           const int32_t* __restrict__ lens) {
    constexpr int CPL = D / 32;
    const int b = blockIdx.z, h = blockIdx.y;
    const int L = lens[b];
    const int n = cu_new[b + 1] - cu_new[b];
    const int w0 = max(L, L + n - p.W);
    const int pos = w0 + blockIdx.x * 4 + (threadIdx.x >> 5);
    if (pos >= L + n || n <= 0) return;
    const int lane = threadIdx.x & 31;
    float kx[CPL], vx[CPL];
    size_t off = (size_t(cu_new[b] + pos - L) * p.hkv + h) * D;
    load_row<D>(k_new, in_bf16, off, lane, kx);
    load_row<D>(v_new, in_bf16, off, lane, vx);
    size_t wo = win_off(p, b, h, pos) + lane * CPL;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        p.k_win[wo + i] = __float2bfloat16_rn(kx[i]);
        p.v_win[wo + i] = __float2bfloat16_rn(vx[i]);
    }
}

// Appends of at most kSmallAppend tokens per sequence, no more than the
// window (the decode step), in one launch: one CTA per (kv-head, sequence),
// one warp per job.  With n <= W every position leaving the ring is older
// than L, and the slot it frees receives position pos + W of this call, so a
// quantize job reads the old row, writes the new token into the same slot,
// then quantizes the old row.  Ring positions below W (slots that held
// nothing) are write-only jobs.  Value codes of one channel share 32-bit
// words across positions: they are merged with atomic and/or, which needs no
// read round trip and leaves the other positions' bits alone.
constexpr int kSmallAppend = 8;

template <int D>
__global__ void __launch_bounds__(128) append_small_kernel(Params p, const void* __restrict__ k_new,
                                                           const void* __restrict__ v_new, int in_bf16,
                                                           const int32_t* __restrict__ cu_new,
                                                           const int32_t* __restrict__ lens) {
    constexpr int CPL = D / 32;
    // a decode launched next as this launch's programmatic dependent may start
    // now: it reads nothing this kernel writes before it waits for its results
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int h = blockIdx.x, b = blockIdx.y;
    const int L = lens[b];
    const int c0 = cu_new[b], n = cu_new[b + 1] - c0;
    if (n <= 0 || L < 0) return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int q0, q1, nd;
    if (p.W > 0) {
        q0 = max(0, L - p.W);
        q1 = max(0, L + n - p.W);
        nd = max(0, min(L + n, p.W) - L);        // ring positions whose slot held nothing
    } else {
        q0 = L;
        q1 = L + n;
        nd = 0;
    }
    const int nq = q1 - q0;
    for (int job = warp; job < nq + nd; job += 4) {
        if (job >= nq) {                             // write-only ring job
            const int pos = L + (job - nq);
            float kx[CPL], vx[CPL];
            const size_t off = (size_t(c0 + pos - L) * p.hkv + h) * D;
            load_row<D>(k_new, in_bf16, off, lane, kx);
            load_row<D>(v_new, in_bf16, off, lane, vx);
            const size_t wo = win_off(p, b, h, pos) + lane * CPL;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                p.k_win[wo + i] = __float2bfloat16_rn(kx[i]);
                p.v_win[wo + i] = __float2bfloat16_rn(vx[i]);
            }
            continue;
        }
        const int pos = q0 + job;
        const int page = phys_page(p, b, pos / kPage);   // issued with the row loads below
        float kx[CPL], vx[CPL];
        if (p.W > 0) {                               // pos < L: the row is in the ring
            const size_t off = win_off(p, b, h, pos);
            load_row<D>(p.k_win, 1, off, lane, kx);
            load_row<D>(p.v_win, 1, off, lane, vx);
            // the new token pos + W takes over the slot
            float nk[CPL], nv[CPL];
            const size_t noff = (size_t(c0 + pos + p.W - L) * p.hkv + h) * D;
            load_row<D>(k_new, in_bf16, noff, lane, nk);
            load_row<D>(v_new, in_bf16, noff, lane, nv);
            const size_t wo = off + lane * CPL;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                p.k_win[wo + i] = __float2bfloat16_rn(nk[i]);
                p.v_win[wo + i] = __float2bfloat16_rn(nv[i]);
            }
        } else {
            const size_t off = (size_t(c0 + pos - L) * p.hkv + h) * D;
            load_row<D>(k_new, in_bf16, off, lane, kx);
            load_row<D>(v_new, in_bf16, off, lane, vx);
        }
        if (page < 0) continue;
        if (p.rotate) rotate_warp<D>(kx, p.signs, lane);
        const int slot = pos % kPage;
        // ---- keys: token row and metadata
        uint32_t kc[CPL];
        const uint32_t km = quantize_warp<D>(kx, p.kg, p.kb, kc);
        if ((lane * CPL) % p.kg == 0) k_meta_row(p, page, h, slot)[(lane * CPL) / p.kg] = km;
        uint32_t bitsv = 0;
#pragma unroll
        for (int i = 0; i < CPL; ++i) bitsv |= kc[i] << (p.kb * i);
        const int lane_bits = CPL * p.kb;            // <= 32
        const int lpw = 32 / lane_bits;              // lanes per 32-bit word
        bitsv <<= (lane % lpw) * lane_bits;
        for (int o = 1; o < lpw; o <<= 1) bitsv |= __shfl_xor_sync(FULL, bitsv, o);
        if (lane % lpw == 0) *k_word(p, page, h, slot, lane / lpw) = bitsv;
        // ---- values: metadata per token, codes merged into the channel words
        uint32_t vc[CPL];
        const uint32_t vm = quantize_warp<D>(vx, p.vg, p.vb, vc);
        if ((lane * CPL) % p.vg == 0) v_meta_row(p, page, h, slot)[(lane * CPL) / p.vg] = vm;
        const int per = 32 / p.vb;
        const uint32_t fmask = (1u << p.vb) - 1u;
        const int shift = p.vb * (slot % per);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            uint32_t* word = v_word(p, page, h, lane * CPL + i, slot / per);
            atomicAnd(word, ~(fmask << shift));
            atomicOr(word, (vc[i] & fmask) << shift);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(128) rotate_rows_kernel(Params p, const void* __restrict__ k, int in_bf16,
                                                          int rows, float* __restrict__ out) {
    constexpr int CPL = D / 32;
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31;
    float x[CPL];
    load_row<D>(k, in_bf16, size_t(row) * D, lane, x);
    rotate_warp<D>(x, p.signs, lane);
#pragma unroll
    for (int i = 0; i < CPL; ++i) out[size_t(row) * D + lane * CPL + i] = x[i];
}

// Reconstruction: one warp per (position, kv-head); quantized positions give
// fmaf(code, scale, zero), window positions their bf16 value.
template <int D>
__global__ void __launch_bounds__(128) dequantize_kernel(Params p, const int32_t* __restrict__ lens,
                                                         int max_len, float* __restrict__ k_out,
                                                         float* __restrict__ v_out) {
    constexpr int CPL = D / 32;
    const int b = blockIdx.z, h = blockIdx.y;
    const int pos = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int L = min(lens[b], max_len);
    if (pos >= L) return;
    const int lane = threadIdx.x & 31;
    float* ko = k_out + ((size_t(b) * p.hkv + h) * max_len + pos) * D + lane * CPL;
    float* vo = v_out + ((size_t(b) * p.hkv + h) * max_len + pos) * D + lane * CPL;
    if (pos >= lens[b] - p.W) {
        size_t off = win_off(p, b, h, pos) + lane * CPL;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            ko[i] = __bfloat162float(p.k_win[off + i]);
            vo[i] = __bfloat162float(p.v_win[off + i]);
        }
        return;
    }
    const int page = phys_page(p, b, pos / kPage);
    if (page < 0) return;
    const int slot = pos % kPage;
    const uint32_t* kmr = k_meta_row(p, page, h, slot);
    const uint32_t* vmr = v_meta_row(p, page, h, slot);
    const int kper = 32 / p.kb, vper = 32 / p.vb;
    const uint32_t kmask = (1u << p.kb) - 1u, vmask = (1u << p.vb) - 1u;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int j = lane * CPL + i;
        uint32_t kc = (*k_word(p, page, h, slot, j / kper) >> (p.kb * (j % kper))) & kmask;
        float2 km = meta_f2(kmr[j / p.kg]);
        ko[i] = __fmaf_rn((float)kc, km.x, km.y);
        uint32_t vc = (*v_word(p, page, h, j, slot / vper) >> (p.vb * (slot % vper))) & vmask;
        float2 vm = meta_f2(vmr[j / p.vg]);
        vo[i] = __fmaf_rn((float)vc, vm.x, vm.y);
    }
}

}  // namespace

bool append_is_one_launch(const Params& p, int max_new) {
    return max_new >= 1 && p.batch > 0 && max_new <= kSmallAppend && (p.W == 0 || max_new <= p.W);
}

cudaError_t launch_quantize_append(const Params& p, const void* k_new, const void* v_new, int in_bf16,
                                   const int32_t* cu_new, const int32_t* lens, int max_new,
                                   cudaStream_t s) {
    if (max_new <= 0 || p.batch <= 0) return cudaSuccess;
    if (append_is_one_launch(p, max_new)) {
        const dim3 sgrid(p.hkv, p.batch);
        if (p.d == 128) append_small_kernel<128><<<sgrid, 128, 0, s>>>(p, k_new, v_new, in_bf16, cu_new, lens);
        else append_small_kernel<64><<<sgrid, 128, 0, s>>>(p, k_new, v_new, in_bf16, cu_new, lens);
        return cudaGetLastError();
    }
    dim3 grid(max_new / 32 + 2, p.hkv, p.batch);
    if (p.d == 128) quantize_pages_kernel<128><<<grid, 128, 0, s>>>(p, k_new, v_new, in_bf16, cu_new, lens);
    else quantize_pages_kernel<64><<<grid, 128, 0, s>>>(p, k_new, v_new, in_bf16, cu_new, lens);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || p.W <= 0) return e;
    const int wn = max_new < p.W ? max_new : p.W;
    dim3 wgrid((wn + 3) / 4, p.hkv, p.batch);
    if (p.d == 128) window_write_kernel<128><<<wgrid, 128, 0, s>>>(p, k_new, v_new, in_bf16, cu_new, lens);
    else window_write_kernel<64><<<wgrid, 128, 0, s>>>(p, k_new, v_new, in_bf16, cu_new, lens);
    return cudaGetLastError();
}

cudaError_t launch_rotate_keys(const Params& p, const void* k, int in_bf16, int rows, float* out,
                               cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    dim3 grid((rows + 3) / 4);
    if (p.d == 128) rotate_rows_kernel<128><<<grid, 128, 0, s>>>(p, k, in_bf16, rows, out);
    else rotate_rows_kernel<64><<<grid, 128, 0, s>>>(p, k, in_bf16, rows, out);
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const Params& p, const int32_t* lens, int max_len, float* k_out,
                              float* v_out, cudaStream_t s) {
    if (max_len <= 0 || p.batch <= 0) return cudaSuccess;
    dim3 grid((max_len + 3) / 4, p.hkv, p.batch);
    if (p.d == 128) dequantize_kernel<128><<<grid, 128, 0, s>>>(p, lens, max_len, k_out, v_out);
    else dequantize_kernel<64><<<grid, 128, 0, s>>>(p, lens, max_len, k_out, v_out);
    return cudaGetLastError();
}

}  // namespace kvq

// Decode attention over the quantized cache on the 5th-generation tensor
// cores (tcgen05, sm_100a), head_dim 128, key groups of 32 channels, value
// groups of 128 channels, any bit widths in {1, 2, 4, 8}.
//
// Attention ("Kuantisasi KV cache mengganggu attention ...", section "Error
// pada key masuk sebelum softmax"): s = q K^T * sm_scale, a = softmax(s),
// o = a V, with dequantization fused into the kernel (section "Pertumbuhan
// cache mengubah trade pada serving").  With x^ = c*scale + zero per group:
//   q . k^ = sum_groups ( scale * (q . c)_group + zero * (sum q)_group )
//   o      = sum_t (p_t scale_t) c_t + sum_t p_t zero_t
// The integer codes are exact in bf16, so both contractions run on the
// tensor cores over the raw codes; scales, zero points and the softmax are
// applied in fp32 around them.
//
// One CTA (4 warps, thread i <-> tensor-memory lane i) walks 128-token tiles
// (two 64-token pages) of one (sequence, kv-head, split):
//   1. the tile's pages are staged into shared memory by 1-D bulk copies
//      (TMA engine) two tiles ahead, completion on an mbarrier;
//   2. thread t unpacks token t's key codes to bf16 and stores them into
//      tensor memory (A operand, M = 128 tokens, K = 128 channels);
//   3. one thread issues tcgen05.mma against the query held in shared memory
//      as a block-diagonal B operand: column (head r, key group, hi/lo half)
//      holds the query's channels of that group only, so the accumulator
//      gives every group's partial dot product (the query is split into a
//      bf16 high part and a bf16 remainder, ~16 significant bits);
//   4. thread t applies scale/zero per group, the online softmax (tile max
//      across the 4 warps), and writes P' = p * value_scale (bf16 high +
//      remainder) into shared memory as the B operand of the second MMA;
//   5. thread j unpacks value channel j's 128 token codes (values are stored
//      channel-major) into tensor memory (A operand, M = 128 channels,
//      K = 128 tokens); the ·V MMA accumulates into a tensor-memory
//      accumulator that is rescaled when the running max moves.
// The bf16 window tokens of the sequence are processed on CUDA cores by the
// last split of each (sequence, kv-head).  Every wait is bounded.
#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_tc_ptx.cuh"

namespace kvq {

// number of bounded waits that expired (diagnostic; 0 in normal operation)
__device__ unsigned int g_tc_wait_timeouts;

namespace {

using namespace ptx;

constexpr int D = 128;
constexpr int kStages = 2;
constexpr int kKGroups = 4;            // key groups of 32 channels
constexpr int COL_A = 0;               // operand A (keys, then values): 64 columns
constexpr int COL_S = 64;              // score accumulator
constexpr int CS_P = 16 * 16 + 16;     // chunk stride of the P' operand (16 rows, padded)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr unsigned FULL = 0xffffffffu;

struct TcShared {
    uint64_t full[kStages];
    uint64_t mma_s;
    uint64_t mma_o;
    uint32_t tmem_base;
    int abort;
    float red[4][kMaxGqa];
    float red2[4][kMaxGqa];
    float qsum[kMaxGqa][kKGroups];
};

struct TcGeom {
    int kc, km, vc, vm;        // bytes per page (one kv-head) of each array
    int stage;                 // bytes per stage (two pages)
    int off_qf, off_qb, off_pb, off_st, total;
    int cs_q;                  // chunk stride of the query operand
};

__host__ __device__ inline TcGeom tc_geom(const Params& p, int ns, int min_total) {
    TcGeom g{};
    g.kc = kPage * p.krow_bytes;
    g.km = kPage * p.nkg * 4;
    g.vc = p.d * p.vchan_bytes;
    g.vm = kPage * p.nvg * 4;
    g.stage = (2 * (g.kc + g.km + g.vc + g.vm) + 127) & ~127;
    g.cs_q = ns * 16 + 16;
    g.off_qf = 1024;
    g.off_qb = g.off_qf + kMaxGqa * D * 4;
    g.off_pb = g.off_qb + 16 * g.cs_q;
    g.off_st = (g.off_pb + 16 * CS_P + 127) & ~127;
    g.total = g.off_st + kStages * g.stage;
    if (g.total < min_total) g.total = min_total;
    return g;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

// ---------------------------------------------------------------- unpacking
// A 32-bit word of b-bit codes becomes 16/b bf16x2 registers; register k
// holds codes (k, k + 16/b): low half the first.  Codes are exact small
// integers: bits are placed into the mantissa of bf16 128.0 (0x4300), the
// offset (and a power-of-two position scale) removed with one exact fma.
template <int S>
__device__ __forceinline__ uint32_t fix_bf16(uint32_t x) {
    __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162 a = __float2bfloat162_rn(1.0f / float(1 << S));
    const __nv_bfloat162 c = __float2bfloat162_rn(-128.0f / float(1 << S));
    __nv_bfloat162 r = __hfma2(v, a, c);
    return *reinterpret_cast<uint32_t*>(&r);
}

constexpr uint32_t kMagic = 0x43004300u;

template <int B>
struct Unpack;

template <>
struct Unpack<4> {
    __device__ static __forceinline__ void word(uint32_t w, uint32_t* o) {
        o[0] = fix_bf16<0>((w & 0x000F000Fu) | kMagic);
        o[1] = fix_bf16<3>(((w >> 1) & 0x00780078u) | kMagic);
        o[2] = fix_bf16<3>(((w >> 5) & 0x00780078u) | kMagic);
        o[3] = fix_bf16<3>(((w >> 9) & 0x00780078u) | kMagic);
    }
};
template <>
struct Unpack<2> {
    __device__ static __forceinline__ void word(uint32_t w, uint32_t* o) {
        o[0] = fix_bf16<0>((w & 0x00030003u) | kMagic);
        o[1] = fix_bf16<2>((w & 0x000C000Cu) | kMagic);
        o[2] = fix_bf16<4>((w & 0x00300030u) | kMagic);
        const uint32_t w6 = w >> 6;
        o[3] = fix_bf16<0>((w6 & 0x00030003u) | kMagic);
        o[4] = fix_bf16<2>((w6 & 0x000C000Cu) | kMagic);
        o[5] = fix_bf16<4>((w6 & 0x00300030u) | kMagic);
        const uint32_t w12 = w >> 12;
        o[6] = fix_bf16<0>((w12 & 0x00030003u) | kMagic);
        o[7] = fix_bf16<2>((w12 & 0x000C000Cu) | kMagic);
    }
};
template <>
struct Unpack<1> {
    __device__ static __forceinline__ void word(uint32_t w, uint32_t* o) {
        o[0] = fix_bf16<0>((w & 0x00010001u) | kMagic);
        o[1] = fix_bf16<1>((w & 0x00020002u) | kMagic);
        o[2] = fix_bf16<2>((w & 0x00040004u) | kMagic);
        o[3] = fix_bf16<3>((w & 0x00080008u) | kMagic);
        o[4] = fix_bf16<4>((w & 0x00100010u) | kMagic);
        o[5] = fix_bf16<5>((w & 0x00200020u) | kMagic);
        o[6] = fix_bf16<6>((w & 0x00400040u) | kMagic);
        const uint32_t w7 = w >> 7;
        o[7] = fix_bf16<0>((w7 & 0x00010001u) | kMagic);
        o[8] = fix_bf16<1>((w7 & 0x00020002u) | kMagic);
        o[9] = fix_bf16<2>((w7 & 0x00040004u) | kMagic);
        o[10] = fix_bf16<3>((w7 & 0x00080008u) | kMagic);
        o[11] = fix_bf16<4>((w7 & 0x00100010u) | kMagic);
        o[12] = fix_bf16<5>((w7 & 0x00200020u) | kMagic);
        o[13] = fix_bf16<6>((w7 & 0x00400040u) | kMagic);
        const uint32_t w14 = w >> 14;
        o[14] = fix_bf16<0>((w14 & 0x00010001u) | kMagic);
        o[15] = fix_bf16<1>((w14 & 0x00020002u) | kMagic);
    }
};
template <>
struct Unpack<8> {
    __device__ static __forceinline__ float byte_f(uint32_t w, uint32_t sel) {
        // float with mantissa = the selected byte, exponent of 2^23; minus 2^23
        return __uint_as_float(__byte_perm(w, 0x4B000000u, sel)) - 8388608.0f;
    }
    __device__ static __forceinline__ void word(uint32_t w, uint32_t* o) {
        __nv_bfloat162 a = __floats2bfloat162_rn(byte_f(w, 0x7440u), byte_f(w, 0x7442u));
        __nv_bfloat162 b = __floats2bfloat162_rn(byte_f(w, 0x7441u), byte_f(w, 0x7443u));
        o[0] = *reinterpret_cast<uint32_t*>(&a);
        o[1] = *reinterpret_cast<uint32_t*>(&b);
    }
};

// position (along the MMA K dimension) of element i of a packed run, and
// the element at a K position: inverse permutations of the unpack order
__host__ __device__ __forceinline__ int kpos_of(int i, int bits) {
    const int per = 32 / bits, half = per / 2;
    const int w = i / per, r = i % per;
    return w * per + 2 * (r % half) + r / half;
}
__host__ __device__ __forceinline__ int elem_at(int pos, int bits) {
    const int per = 32 / bits, half = per / 2;
    const int w = pos / per, r = pos % per;
    return w * per + (r >> 1) + (r & 1) * half;
}
// byte offset of element (row n, K position pos) in a K-major B operand
// stored as [k step][half][row][8 x bf16] with chunk stride cs
__device__ __forceinline__ int b_off(int n, int pos, int cs) {
    return ((pos >> 4) * 2 + ((pos >> 3) & 1)) * cs + n * 16 + (pos & 7) * 2;
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// ------------------------------------------------------------- window part
// bf16 window tokens [Lq, L) on CUDA cores; writes one partial (m, l, o).
__device__ void window_partial(const Params& p, int b, int h, int Lq, int L, const float (*qf)[D],
                               float* pw /* [kMaxGqa][128] */, TcShared& sh, float scale_log2,
                               float* ws_o, float* ws_ml, size_t row0, int slots, int slot) {
    const int g = p.g, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float mrun[kMaxGqa], lpart[kMaxGqa], o[kMaxGqa];
#pragma unroll
    for (int r = 0; r < kMaxGqa; ++r) {
        mrun[r] = -INFINITY;
        lpart[r] = 0.0f;
        o[r] = 0.0f;
    }
    for (int cb = Lq; cb < L; cb += 128) {
        const int pos = cb + tid;
        const bool valid = pos < L;
        float s[kMaxGqa];
#pragma unroll
        for (int r = 0; r < kMaxGqa; ++r) s[r] = 0.0f;
        if (valid) {
            const uint4* kr = reinterpret_cast<const uint4*>(p.k_win + win_off(p, b, h, pos));
            uint4 krow[D / 8];
#pragma unroll
            for (int c = 0; c < D / 8; ++c) krow[c] = kr[c];
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 u = krow[c];
                const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[e]));
                    const int j = c * 8 + e * 2;
#pragma unroll
                    for (int r = 0; r < kMaxGqa; ++r)
                        if (r < g) s[r] = fmaf(kv.y, qf[r][j + 1], fmaf(kv.x, qf[r][j], s[r]));
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kMaxGqa; ++r) {
            s[r] = (valid && r < g) ? s[r] * scale_log2 : -INFINITY;
            const float m = warp_max(s[r]);
            if (lane == 0) sh.red[warp][r] = m;
        }
        __syncthreads();
        float alpha[kMaxGqa];
#pragma unroll
        for (int r = 0; r < kMaxGqa; ++r) {
            const float tmax = fmaxf(fmaxf(sh.red[0][r], sh.red[1][r]), fmaxf(sh.red[2][r], sh.red[3][r]));
            const float mnew = fmaxf(mrun[r], tmax);
            const float mu = (mnew == -INFINITY) ? 0.0f : mnew;
            alpha[r] = exp2f(mrun[r] - mu);
            mrun[r] = mnew;
            const float pr = exp2f(s[r] - mu);
            lpart[r] = fmaf(lpart[r], alpha[r], pr);
            if (r < g) pw[r * 128 + tid] = pr;
        }
        __syncthreads();
        const int n = min(128, L - cb);
#pragma unroll
        for (int r = 0; r < kMaxGqa; ++r) o[r] *= alpha[r];
        // value column `tid` of the ring, 16 independent loads in flight
        const __nv_bfloat16* vcol = p.v_win + (size_t(b) * p.hkv + h) * size_t(p.W) * D + tid;
        int t = 0;
        for (; t + 16 <= n; t += 16) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = __bfloat162float(vcol[size_t((cb + t + k) % p.W) * D]);
#pragma unroll
            for (int k = 0; k < 16; ++k)
#pragma unroll
                for (int r = 0; r < kMaxGqa; ++r)
                    if (r < g) o[r] = fmaf(pw[r * 128 + t + k], v[k], o[r]);
        }
        for (; t < n; ++t) {
            const float v = __bfloat162float(vcol[size_t((cb + t) % p.W) * D]);
#pragma unroll
            for (int r = 0; r < kMaxGqa; ++r)
                if (r < g) o[r] = fmaf(pw[r * 128 + t], v, o[r]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < kMaxGqa; ++r) {
        const float l = warp_sum(lpart[r]);
        if (lane == 0) sh.red2[warp][r] = l;
    }
    __syncthreads();
    for (int r = 0; r < g; ++r) {
        ws_o[(row0 + size_t(r) * slots + slot) * D + tid] = o[r];
        if (tid == 0) {
            const float l = sh.red2[0][r] + sh.red2[1][r] + sh.red2[2][r] + sh.red2[3][r];
            ws_ml[(row0 + size_t(r) * slots + slot) * 2 + 0] = mrun[r];
            ws_ml[(row0 + size_t(r) * slots + slot) * 2 + 1] = l;
        }
    }
    __syncthreads();
}

__device__ void empty_partial(int g, float* ws_o, float* ws_ml, size_t row0, int slots, int slot) {
    for (int r = 0; r < g; ++r) {
        ws_o[(row0 + size_t(r) * slots + slot) * D + threadIdx.x] = 0.0f;
        if (threadIdx.x == 0) {
            ws_ml[(row0 + size_t(r) * slots + slot) * 2 + 0] = -INFINITY;
            ws_ml[(row0 + size_t(r) * slots + slot) * 2 + 1] = 0.0f;
        }
    }
}

// ------------------------------------------------------------------ kernel
// grid (splits_q, Hkv, B), 128 threads.  Split s covers quantized pages
// [s*pps, (s+1)*pps); the last split also covers the bf16 window.
template <int KB, int VB, int NS>
__global__ void __launch_bounds__(128, (NS == 32 ? 4 : 2))
decode_tc_kernel(const Params p, const void* __restrict__ q, const int q_bf16, const int32_t* __restrict__ lens,
                 const int max_len, const float scale_log2, float* __restrict__ ws_o, float* __restrict__ ws_ml,
                 const int pps, const int slots, const int window_slot, const TcGeom geo) {
    constexpr int NH = NS / 8;               // heads the score accumulator holds
    constexpr int KW = D * KB / 32;          // words per key row
    constexpr int KREG = 16 / KB;            // bf16x2 registers per key word
    constexpr int VWP = kPage * VB / 32;     // words per value channel per page
    constexpr int VREG = 16 / VB;
    constexpr uint32_t TMEM_COLS = (COL_S + NS + 16 <= 128) ? 128u : 256u;
    constexpr int COL_O = COL_S + NS;
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, NS);
    constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 16);

    extern __shared__ __align__(1024) uint8_t smem[];
    TcShared& sh = *reinterpret_cast<TcShared*>(smem);
    float(*qf)[D] = reinterpret_cast<float(*)[D]>(smem + geo.off_qf);
    uint8_t* qb = smem + geo.off_qb;
    uint8_t* pb = smem + geo.off_pb;
    uint8_t* st = smem + geo.off_st;

    const int b = blockIdx.z, h = blockIdx.y, split = blockIdx.x;
    const int g = p.g, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = max(0, min(lens[b], max_len));
    const int Lq = max(0, L - p.W);
    const int npg = (Lq + kPage - 1) / kPage;
    const int pg0 = split * pps;
    const int pg1 = min(npg, pg0 + pps);
    const int ntiles = pg1 > pg0 ? (pg1 - pg0 + 1) / 2 : 0;
    const bool last = split == (int)gridDim.x - 1;
    const size_t row0 = (size_t(b) * p.hq + size_t(h) * g) * slots;

    // unrotated query, fp32
    for (int i = tid; i < g * D; i += 128) {
        const size_t off = (size_t(b) * p.hq + size_t(h) * g + i / D) * D + (i % D);
        qf[i / D][i % D] = q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[off])
                                  : reinterpret_cast<const float*>(q)[off];
    }

    if (ntiles == 0) {
        empty_partial(g, ws_o, ws_ml, row0, slots, split);
    } else {
        // ---------------------------------------------------------- set-up
        if (tid == 0) {
            for (int s = 0; s < kStages; ++s) mbar_init(&sh.full[s], 1);
            mbar_init(&sh.mma_s, 1);
            mbar_init(&sh.mma_o, 1);
            mbar_fence_init();
            sh.abort = 0;
        }
        if (warp == 0) {
            tmem_alloc(&sh.tmem_base, TMEM_COLS);
            tmem_relinquish();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        const uint32_t tbase = sh.tmem_base;
        const uint32_t lane_off = uint32_t(warp * 32) << 16;

        auto issue_tile = [&](int stage, int tile) {
            uint8_t* sb = st + stage * geo.stage;
            const void* src[8];
            void* dst[8];
            uint32_t len[8];
            int n = 0;
            uint32_t bytes = 0;
            for (int pp = 0; pp < 2; ++pp) {
                const int lp = pg0 + 2 * tile + pp;
                if (lp >= pg1) break;
                const int pg = phys_page(p, b, lp);
                if (pg < 0) continue;
                const size_t ph = size_t(pg) * p.hkv + h;
                src[n] = p.k_codes + ph * geo.kc;      dst[n] = sb + pp * geo.kc;                  len[n++] = geo.kc;
                src[n] = reinterpret_cast<const uint8_t*>(p.k_meta) + ph * geo.km;
                dst[n] = sb + 2 * geo.kc + pp * geo.km;                                              len[n++] = geo.km;
                src[n] = p.v_codes + ph * geo.vc;
                dst[n] = sb + 2 * (geo.kc + geo.km) + pp * geo.vc;                                   len[n++] = geo.vc;
                src[n] = reinterpret_cast<const uint8_t*>(p.v_meta) + ph * geo.vm;
                dst[n] = sb + 2 * (geo.kc + geo.km + geo.vc) + pp * geo.vm;                          len[n++] = geo.vm;
                bytes += geo.kc + geo.km + geo.vc + geo.vm;
            }
            fence_proxy_async();
            mbar_arrive_expect_tx(&sh.full[stage], bytes);
            for (int i = 0; i < n; ++i) bulk_g2s(dst[i], src[i], len[i], &sh.full[stage]);
        };
        if (tid == 0) {
            for (int s = 0; s < kStages && s < ntiles; ++s) issue_tile(s, s);
        }

        // query operand: rotated query (when keys are rotated) as bf16 hi +
        // bf16 remainder, block-diagonal over the key groups
        float* qr = reinterpret_cast<float*>(pb);              // scratch [g][D] before P' exists
        __syncthreads();                                        // qf complete
        for (int r = warp; r < g; r += 4) {
            float x[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) x[c] = qf[r][lane * 4 + c];
            if (p.rotate) rotate_warp<D>(x, p.signs, lane);
#pragma unroll
            for (int c = 0; c < 4; ++c) qr[r * D + lane * 4 + c] = x[c];
        }
        __syncthreads();
        for (int i = tid; i < g * kKGroups; i += 128) {
            const int r = i / kKGroups, grp = i % kKGroups;
            float s = 0.0f;
            for (int j = grp * 32; j < grp * 32 + 32; ++j) s += qr[r * D + j];
            sh.qsum[r][grp] = s;
        }
        for (int e = tid; e < NS * D; e += 128) {
            const int n = e / D, pos = e % D;
            uint16_t v = 0;
            const int r = n >> 3, grp = (n >> 1) & 3, hl = n & 1;
            if (r < g) {
                const int j = elem_at(pos, KB);
                if ((j >> 5) == grp) {
                    const float x = qr[r * D + j];
                    const float hi = __bfloat162float(__float2bfloat16_rn(x));
                    v = hl ? bf16_bits(x - hi) : bf16_bits(x);
                }
            }
            *reinterpret_cast<uint16_t*>(qb + b_off(n, pos, geo.cs_q)) = v;
        }
        __syncthreads();                                        // qr reads done
        for (int i = tid; i < 16 * CS_P / 4; i += 128) reinterpret_cast<uint32_t*>(pb)[i] = 0u;
        fence_proxy_async();
        __syncthreads();

        float mrun[NH], lpart[NH], pzpart[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            mrun[r] = -INFINITY;
            lpart[r] = 0.0f;
            pzpart[r] = 0.0f;
        }
        const int pp_t = tid >> 6, slot_t = tid & 63;           // token role
        const int kpos_t = pp_t * kPage + kpos_of(slot_t, VB);   // its position along the ·V K dim
        bool ok = true;

        for (int i = 0; i < ntiles; ++i) {
            const int stage = i % kStages;
            const uint8_t* sb = st + stage * geo.stage;
            if (!mbar_wait(&sh.full[stage], (i / kStages) & 1, kWaitNs)) ok = false;
            // ---- token role: key codes and metadata of token t
            const int lp = pg0 + 2 * i + pp_t;
            const int pos = lp * kPage + slot_t;
            const bool valid = lp < pg1 && pos < Lq && phys_page(p, b, lp) >= 0;
            uint32_t ka[64];
            {
                const uint4* kr = reinterpret_cast<const uint4*>(sb + pp_t * geo.kc + slot_t * (KW * 4));
#pragma unroll
                for (int c = 0; c < KW / 4; ++c) {
                    const uint4 u = kr[c];
                    Unpack<KB>::word(u.x, &ka[(4 * c + 0) * KREG]);
                    Unpack<KB>::word(u.y, &ka[(4 * c + 1) * KREG]);
                    Unpack<KB>::word(u.z, &ka[(4 * c + 2) * KREG]);
                    Unpack<KB>::word(u.w, &ka[(4 * c + 3) * KREG]);
                }
            }
            float ksc[kKGroups], kzp[kKGroups];
            {
                const uint4 m4 = *reinterpret_cast<const uint4*>(sb + 2 * geo.kc + pp_t * geo.km + slot_t * 16);
                const uint32_t mw[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                for (int grp = 0; grp < kKGroups; ++grp) {
                    const float2 f = meta_f2(mw[grp]);
                    ksc[grp] = f.x;
                    kzp[grp] = f.y;
                }
            }
            float vsc = 0.0f, vzp = 0.0f;
            if (valid) {
                const float2 f = meta_f2(*reinterpret_cast<const uint32_t*>(
                    sb + 2 * (geo.kc + geo.km + geo.vc) + pp_t * geo.vm + slot_t * 4));
                vsc = f.x;
                vzp = f.y;
            }
            // operand A (keys) may be overwritten once the previous ·V MMA is done
            if (i > 0 && !mbar_wait(&sh.mma_o, (i - 1) & 1, kWaitNs)) ok = false;
            tc_fence_after();
            tmem_st64(tbase + lane_off + COL_A, ka);
            tc_wait_st();
            tc_fence_before();
            if (!ok) sh.abort = 1;
            __syncthreads();                                                      // S1
            if (sh.abort) break;
            if (tid == 0) {
                tc_fence_after();
                const uint32_t qbase = smem_u32(qb);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    tc_mma_ts(tbase + COL_S, tbase + COL_A + ks * 8,
                              smem_desc(qbase + ks * 2 * geo.cs_q, geo.cs_q, 128), IDESC_S, ks > 0);
                tc_commit(&sh.mma_s);
            }
            // ---- channel role: value codes of channel j = tid for the tile's tokens
            uint32_t va[64];
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
                const uint32_t* vr = reinterpret_cast<const uint32_t*>(sb + 2 * (geo.kc + geo.km) + pp * geo.vc +
                                                                       tid * (VWP * 4));
#pragma unroll
                for (int w = 0; w < VWP; ++w) Unpack<VB>::word(vr[w], &va[pp * 32 + w * VREG]);
            }
            if (!mbar_wait(&sh.mma_s, i & 1, kWaitNs)) ok = false;
            tc_fence_after();
            uint32_t ds[NS];
#pragma unroll
            for (int c = 0; c < NS / 16; ++c) tmem_ld16(tbase + lane_off + COL_S + c * 16,
                                                        *reinterpret_cast<uint32_t(*)[16]>(&ds[c * 16]));
            tc_wait_ld();
            tmem_st64(tbase + lane_off + COL_A, va);                              // keys no longer needed
            // ---- scores and tile max
            float s[NH];
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                float acc = 0.0f;
#pragma unroll
                for (int grp = 0; grp < kKGroups; ++grp) {
                    const float dot = __uint_as_float(ds[r * 8 + 2 * grp]) + __uint_as_float(ds[r * 8 + 2 * grp + 1]);
                    acc = fmaf(ksc[grp], dot, fmaf(kzp[grp], sh.qsum[r < g ? r : 0][grp], acc));
                }
                s[r] = (valid && r < g) ? acc * scale_log2 : -INFINITY;
                const float m = warp_max(s[r]);
                if (lane == 0) sh.red[warp][r] = m;
            }
            if (!ok) sh.abort = 1;
            __syncthreads();                                                      // S2
            if (sh.abort) break;
            if (tid == 0 && i + kStages < ntiles) issue_tile(stage, i + kStages);
            // ---- online softmax, P' = p * value scale (bf16 hi + remainder)
            float alpha[NH];
            bool moved = false;
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                const float tmax = fmaxf(fmaxf(sh.red[0][r], sh.red[1][r]), fmaxf(sh.red[2][r], sh.red[3][r]));
                const float mnew = fmaxf(mrun[r], tmax);
                const float mu = (mnew == -INFINITY) ? 0.0f : mnew;
                alpha[r] = exp2f(mrun[r] - mu);
                moved |= (mnew != mrun[r]);
                mrun[r] = mnew;
                const float pr = exp2f(s[r] - mu);
                lpart[r] = fmaf(lpart[r], alpha[r], pr);
                pzpart[r] = fmaf(pzpart[r], alpha[r], pr * vzp);
                const float pv = pr * vsc;
                const float hi = __bfloat162float(__float2bfloat16_rn(pv));
                if (r < g) {
                    *reinterpret_cast<uint16_t*>(pb + b_off(2 * r, kpos_t, CS_P)) = bf16_bits(pv);
                    *reinterpret_cast<uint16_t*>(pb + b_off(2 * r + 1, kpos_t, CS_P)) = bf16_bits(pv - hi);
                }
            }
            // running max moved: rescale the ·V accumulator (no MMA in flight on it)
            if (i > 0 && moved) {
                uint32_t o[16];
                tmem_ld16(tbase + lane_off + COL_O, o);
                tc_wait_ld();
#pragma unroll
                for (int n = 0; n < 16; ++n) o[n] = __float_as_uint(__uint_as_float(o[n]) * alpha[(n >> 1) < NH ? (n >> 1) : 0]);
                tmem_st16(tbase + lane_off + COL_O, o);
            }
            tc_wait_st();
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();                                                      // S3
            if (tid == 0) {
                tc_fence_after();
                const uint32_t pbase = smem_u32(pb);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    tc_mma_ts(tbase + COL_O, tbase + COL_A + ks * 8, smem_desc(pbase + ks * 2 * CS_P, CS_P, 128),
                              IDESC_O, (i > 0 || ks > 0) ? 1u : 0u);
                tc_commit(&sh.mma_o);
            }
        }
        // ---------------------------------------------------------- epilogue
        const bool aborted = sh.abort != 0;
        if (!aborted && !mbar_wait(&sh.mma_o, (ntiles - 1) & 1, kWaitNs)) ok = false;
        tc_fence_after();
        uint32_t o[16];
        tmem_ld16(tbase + lane_off + COL_O, o);
        tc_wait_ld();
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            const float l = warp_sum(lpart[r]);
            const float z = warp_sum(pzpart[r]);
            if (lane == 0) {
                sh.red[warp][r] = l;
                sh.red2[warp][r] = z;
            }
        }
        __syncthreads();
        const bool bad = aborted || !ok;
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            if (r >= g) continue;
            const float z = sh.red2[0][r] + sh.red2[1][r] + sh.red2[2][r] + sh.red2[3][r];
            const float val = __uint_as_float(o[2 * r]) + __uint_as_float(o[2 * r + 1]) + z;
            ws_o[(row0 + size_t(r) * slots + split) * D + tid] = bad ? NAN : val;
            if (tid == 0) {
                const float l = sh.red[0][r] + sh.red[1][r] + sh.red[2][r] + sh.red[3][r];
                ws_ml[(row0 + size_t(r) * slots + split) * 2 + 0] = bad ? 0.0f : mrun[r];
                ws_ml[(row0 + size_t(r) * slots + split) * 2 + 1] = bad ? NAN : l;
            }
        }
        if (bad && tid == 0) atomicAdd(&g_tc_wait_timeouts, 1u);
        if (aborted) {
            // let copies still in flight land before the shared memory is released
            for (int s = 0; s < kStages; ++s) mbar_wait(&sh.full[s], 0, kWaitNs / 8);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            tmem_dealloc(tbase, TMEM_COLS);
        }
    }
    if (last && p.W > 0) {
        __syncthreads();
        window_partial(p, b, h, Lq, L, qf, reinterpret_cast<float*>(st), sh, scale_log2, ws_o, ws_ml, row0,
                       slots, window_slot);
    }
}

template <int KB, int VB, int NS>
cudaError_t launch_tc_t(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                        float scale_log2, float* ws_o, float* ws_ml, const DecodePlan& pl, cudaStream_t s) {
    constexpr uint32_t cols = (COL_S + NS + 16 <= 128) ? 128u : 256u;
    const int ctas_per_sm = int(512 / cols);
    // shared memory sized so that no more CTAs are resident than tensor memory holds
    const int min_total = (228 * 1024) / (ctas_per_sm + 1) + 1024;
    const TcGeom geo = tc_geom(p, NS, min_total);
    auto kern = decode_tc_kernel<KB, VB, NS>;
    static int configured = 0;
    if (configured < geo.total) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.total);
        if (e != cudaSuccess) return e;
        configured = geo.total;
    }
    dim3 grid(pl.grid_x, p.hkv, p.batch);
    kern<<<grid, 128, geo.total, s>>>(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl.pages_per_split,
                                     pl.total_splits, pl.window_slot, geo);
    return cudaGetLastError();
}

template <int NS>
cudaError_t dispatch_bits(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                          float* wo, float* wml, const DecodePlan& pl, cudaStream_t s) {
    const int key = p.kb * 10 + p.vb;
    switch (key) {
        case 42: return launch_tc_t<4, 2, NS>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 44: return launch_tc_t<4, 4, NS>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 88: return launch_tc_t<8, 8, NS>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 24: return launch_tc_t<2, 4, NS>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 22: return launch_tc_t<2, 2, NS>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 12: return launch_tc_t<1, 2, NS>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

bool tc_supported(const Params& p) {
    if (p.d != D || p.kg != 32 || p.vg != 128 || p.g > kMaxGqa) return false;
    const int key = p.kb * 10 + p.vb;
    return key == 42 || key == 44 || key == 88 || key == 24 || key == 22 || key == 12;
}

int tc_ctas_per_sm(const Params& p) { return p.g <= 4 ? 4 : 2; }

cudaError_t launch_decode_tc(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                             float scale_log2, float* ws_o, float* ws_ml, const DecodePlan& pl, cudaStream_t s) {
    if (p.g <= 4) return dispatch_bits<32>(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl, s);
    return dispatch_bits<64>(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl, s);
}

}  // namespace kvq

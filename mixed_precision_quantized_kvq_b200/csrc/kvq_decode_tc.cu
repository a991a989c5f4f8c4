// Decode attention over the quantized cache on the 5th-generation tensor
// cores (tcgen05, sm_100a), head_dim 128, key groups of 32 channels, value
// groups of 128 channels, bit pairs K/V in {4/2, 4/4, 8/8, 2/4, 2/2, 1/2}.
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
// Warp-specialised pipeline, one CTA per SM, 128-token tiles (two pages):
//   warp 12      TMA: 1-D bulk copies of each tile's pages into a ring of
//                shared-memory stages (mbarrier full / empty per stage);
//   warps 0-3    keys: thread t unpacks token t's codes to exact bf16 and
//                stores them into tensor memory (A operand, M = 128 tokens,
//                K = 128 channels), double buffered;
//   warp 13      MMA: one thread issues the score MMA of tile i (query held
//                in shared memory as a block-diagonal B operand: column
//                (head r, key group, bf16 high / remainder) carries only that
//                group's channels) and the ·V MMA of tile i-1;
//   warps 4-7    softmax: thread t applies scale/zero per group, keeps the
//                running max (reused while scores stay within 2^8 of it; a
//                larger score triggers an exact max and a rescale of the ·V
//                accumulator) and writes P' = p * value_scale as the B
//                operand of the ·V MMA (bf16 high + remainder);
//   warps 8-11   values: thread j unpacks value channel j's 128 token codes
//                (values are stored channel-major) into tensor memory (A
//                operand, M = 128 channels, K = 128 tokens).
// The roles hand buffers to each other through mbarriers only, so unpacking
// tile i+1, the softmax of tile i and the MMAs overlap.  The bf16 window
// tokens of a sequence run through the same pipeline (operands read from the
// window ring, scale 1, zero 0) in the last split.  Every wait is bounded.
#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_tc_ptx.cuh"

namespace kvq {

// number of bounded waits that expired (diagnostic; 0 in normal operation)
__device__ unsigned int g_tc_wait_timeouts;

namespace {

using namespace ptx;

constexpr int D = 128;
constexpr int kMaxStages = 8;
constexpr int kKGroups = 4;            // key groups of 32 channels
constexpr int CS_P = 16 * 16 + 16;     // chunk stride of the P' operand (16 rows, padded)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr unsigned FULL = 0xffffffffu;
constexpr int kMaxPagesPerSplit = 256;
constexpr float kLazyMax = 8.0f;       // reuse the running max while scores exceed it by <= 2^8
constexpr int kThreads = 14 * 32;
// tensor-memory columns
constexpr int COL_AK = 0;              // key operands, 2 x 64
constexpr int COL_AV = 128;            // value operands, 2 x 64
constexpr int COL_S = 256;             // score accumulators, 2 x NS
// ·V accumulator at COL_S + 2*NS, 16 columns

struct TcShared {
    uint64_t full[kMaxStages];     // TMA -> consumers: stage loaded
    uint64_t empty[kMaxStages];    // 12 consumer warps -> TMA: stage read
    uint64_t kfull[2], kfree[2];   // key operand written / consumed by the score MMA
    uint64_t sfull[2], sfree[2];   // score accumulator ready / read
    uint64_t vfull[2], vfree[2];   // value operand written / consumed by the ·V MMA
    uint64_t pfull[2], pfree[2];   // P' operand written / consumed by the ·V MMA
    uint32_t tmem_base;
    int abort;
    int vote[2][4];                // softmax warps: lazy-max votes, per tile parity
    float4 red[2][kMaxGqa];        // softmax warps: per-warp partials
    float4 red2[kMaxGqa];
    float4 qsum[kMaxGqa];          // [head] -> query sums of the 4 key groups
    int pages[kMaxPagesPerSplit];  // physical page of each logical page of the split, -1 if absent
};

struct TcGeom {
    int kc, km, vc, vm;        // bytes per page (one kv-head) of each array
    int stage;                 // bytes per stage (one 128-token tile = two pages)
    int nstages;               // stages in the ring
    int off_qf, off_qr, off_qb, off_pb, off_st, total;
    int cs_q;                  // chunk stride of the query operand
};

__host__ __device__ inline TcGeom tc_geom(const Params& p, int ns, int max_total) {
    TcGeom g{};
    g.kc = kPage * p.krow_bytes;
    g.km = kPage * p.nkg * 4;
    g.vc = p.d * p.vchan_bytes;
    g.vm = kPage * p.nvg * 4;
    g.stage = (2 * (g.kc + g.km + g.vc + g.vm) + 127) & ~127;
    g.cs_q = ns * 16 + 16;
    g.off_qf = (int(sizeof(TcShared)) + 127) & ~127;
    g.off_qr = g.off_qf + kMaxGqa * D * 4;
    g.off_qb = g.off_qr + kMaxGqa * D * 4;               // two variants: rotated / unrotated query
    g.off_pb = g.off_qb + 2 * 16 * g.cs_q;               // two buffers
    g.off_st = (g.off_pb + 2 * 16 * CS_P + 127) & ~127;
    g.nstages = (max_total - g.off_st) / g.stage;
    if (g.nstages > kMaxStages) g.nstages = kMaxStages;
    g.total = g.off_st + g.nstages * g.stage;
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
// bf16 bit patterns (both halves) of 2^-S and -128 * 2^-S
template <int S>
struct FixConst;
template <> struct FixConst<0> { static constexpr uint32_t mul = 0x3F803F80u, add = 0xC300C300u; };
template <> struct FixConst<1> { static constexpr uint32_t mul = 0x3F003F00u, add = 0xC280C280u; };
template <> struct FixConst<2> { static constexpr uint32_t mul = 0x3E803E80u, add = 0xC200C200u; };
template <> struct FixConst<3> { static constexpr uint32_t mul = 0x3E003E00u, add = 0xC180C180u; };
template <> struct FixConst<4> { static constexpr uint32_t mul = 0x3D803D80u, add = 0xC100C100u; };
template <> struct FixConst<5> { static constexpr uint32_t mul = 0x3D003D00u, add = 0xC080C080u; };
template <> struct FixConst<6> { static constexpr uint32_t mul = 0x3C803C80u, add = 0xC000C000u; };

template <int S>
__device__ __forceinline__ uint32_t fix_bf16(uint32_t x) {
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(FixConst<S>::mul), "r"(FixConst<S>::add));
    return r;
}

__device__ __forceinline__ float ex2(float x) {   // 2^x, hardware approximation (flushes subnormals)
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
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


__device__ void empty_partial(int g, float* ws_o, float* ws_ml, size_t row0, int slots, int slot) {
    for (int i = threadIdx.x; i < g * D; i += blockDim.x) {
        const int r = i / D;
        ws_o[(row0 + size_t(r) * slots + slot) * D + (i % D)] = 0.0f;
        if (i % D == 0) {
            ws_ml[(row0 + size_t(r) * slots + slot) * 2 + 0] = -INFINITY;
            ws_ml[(row0 + size_t(r) * slots + slot) * 2 + 1] = 0.0f;
        }
    }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ kernel
// grid (splits_q, Hkv, B), 448 threads, one CTA per SM.  Split s covers
// quantized pages [s*pps, (s+1)*pps); the last split also covers the bf16
// window tokens as further tiles, so every split writes exactly one partial
// (m, l, o) per query head.
template <int KB, int VB, int NS>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const Params p, const void* __restrict__ q, const int q_bf16, const int32_t* __restrict__ lens,
                 const int max_len, const float scale_log2, float* __restrict__ ws_o, float* __restrict__ ws_ml,
                 const int pps, const int slots, const TcGeom geo) {
    constexpr int NH = NS / 8;               // heads the score accumulator holds
    constexpr int KW = D * KB / 32;          // words per key row
    constexpr int KREG = 16 / KB;            // bf16x2 registers per key word
    constexpr int VWP = kPage * VB / 32;     // words per value channel per page
    constexpr int VREG = 16 / VB;
    constexpr int COL_O = COL_S + 2 * NS;
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, NS);
    constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 16);

    extern __shared__ __align__(1024) uint8_t smem[];
    TcShared& sh = *reinterpret_cast<TcShared*>(smem);
    float(*qf)[D] = reinterpret_cast<float(*)[D]>(smem + geo.off_qf);
    float(*qr)[D] = reinterpret_cast<float(*)[D]>(smem + geo.off_qr);
    uint8_t* qb = smem + geo.off_qb;
    uint8_t* pb = smem + geo.off_pb;
    uint8_t* st = smem + geo.off_st;
    const int nst = geo.nstages;

    const int b = blockIdx.z, h = blockIdx.y, split = blockIdx.x;
    const int g = p.g, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = max(0, min(lens[b], max_len));
    const int Lq = max(0, L - p.W);
    const int npg = (Lq + kPage - 1) / kPage;
    const int pg0 = split * pps;
    const int pg1 = min(npg, pg0 + pps);
    const int ntiles = pg1 > pg0 ? (pg1 - pg0 + 1) / 2 : 0;
    const bool last = split == (int)gridDim.x - 1;
    const int nwin = (last && p.W > 0 && L > Lq) ? (L - Lq + 127) / 128 : 0;   // bf16 window tiles
    const int ntot = ntiles + nwin;
    const size_t row0 = (size_t(b) * p.hq + size_t(h) * g) * slots;
    if (ntot == 0) {
        empty_partial(g, ws_o, ws_ml, row0, slots, split);
        return;
    }

    // ------------------------------------------------------------------ set-up
    if (tid == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 12);
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(&sh.kfull[u], 4);
            mbar_init(&sh.kfree[u], 1);
            mbar_init(&sh.sfull[u], 1);
            mbar_init(&sh.sfree[u], 4);
            mbar_init(&sh.vfull[u], 4);
            mbar_init(&sh.vfree[u], 1);
            mbar_init(&sh.pfull[u], 4);
            mbar_init(&sh.pfree[u], 1);
        }
        mbar_fence_init();
        sh.abort = 0;
    }
    if (warp == 0) {
        tmem_alloc(&sh.tmem_base, 512);
        tmem_relinquish();
    }
    for (int i = tid; i < pg1 - pg0; i += kThreads) sh.pages[i] = phys_page(p, b, pg0 + i);
    for (int i = tid; i < g * D; i += kThreads) {            // unrotated query, fp32
        const size_t off = (size_t(b) * p.hq + size_t(h) * g + i / D) * D + (i % D);
        qf[i / D][i % D] = q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[off])
                                  : reinterpret_cast<const float*>(q)[off];
    }
    __syncthreads();
    for (int r = warp; r < g; r += kThreads / 32) {             // rotated query (keys rotated)
        float x[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = qf[r][lane * 4 + c];
        if (p.rotate) rotate_warp<D>(x, p.signs, lane);
#pragma unroll
        for (int c = 0; c < 4; ++c) qr[r][lane * 4 + c] = x[c];
    }
    __syncthreads();
    for (int i = tid; i < g * kKGroups; i += kThreads) {
        const int r = i / kKGroups, grp = i % kKGroups;
        float sum = 0.0f;
        for (int j = grp * 32; j < grp * 32 + 32; ++j) sum += qr[r][j];
        reinterpret_cast<float*>(&sh.qsum[r])[grp] = sum;
    }
    // query operands (bf16 high + remainder, block-diagonal over the key
    // groups, column 8r + 2grp + hl): variant 0 from the rotated query,
    // variant 1 from the unrotated one (window keys of a rotating layout)
    const bool need_unrot = p.rotate && nwin > 0;
    for (int e = tid; e < (need_unrot ? 2 : 1) * D; e += kThreads) {
        const int var = e / D, pos = e % D;
        const int j = elem_at(pos, KB);
        const int grp = j >> 5;
        const float(*src)[D] = var ? qf : qr;
        uint8_t* dst = qb + var * 16 * geo.cs_q;
        for (int n = 0; n < NS; ++n) {
            const int r = n >> 3;
            uint16_t v = 0;
            if (r < g && ((n >> 1) & 3) == grp) {
                const float x = src[r][j];
                const float hi = __bfloat162float(__float2bfloat16_rn(x));
                v = (n & 1) ? bf16_bits(x - hi) : bf16_bits(x);
            }
            *reinterpret_cast<uint16_t*>(dst + b_off(n, pos, geo.cs_q)) = v;
        }
    }
    for (int i = tid; i < 2 * 16 * CS_P / 4; i += kThreads) reinterpret_cast<uint32_t*>(pb)[i] = 0u;
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sh.tmem_base;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;   // this warp's tensor-memory lanes
    const int wslot0 = p.W > 0 ? Lq % p.W : 0;                    // ring slot of position Lq
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        if (!ok || sh.abort) {
            ok = false;
            return;
        }
        if (!mbar_wait(bar, parity, kWaitNs)) {
            ok = false;
            sh.abort = 1;
        }
    };

    if (warp == 12) {
        // ============================================================== TMA
        if (lane == 0) {
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % nst;
                if (i >= nst) wait(&sh.empty[s], ((i / nst) - 1) & 1);
                if (!ok) break;
                uint8_t* sb = st + s * geo.stage;
                const int per_page = geo.kc + geo.km + geo.vc + geo.vm;
                uint32_t bytes = 0;
                for (int pp = 0; pp < 2; ++pp) {
                    const int lp = pg0 + 2 * i + pp;
                    if (lp < pg1 && sh.pages[2 * i + pp] >= 0) bytes += per_page;
                }
                mbar_arrive_expect_tx(&sh.full[s], bytes);
                for (int pp = 0; pp < 2; ++pp) {
                    const int lp = pg0 + 2 * i + pp;
                    if (lp >= pg1) break;
                    const int pg = sh.pages[2 * i + pp];
                    if (pg < 0) continue;
                    const size_t ph = size_t(pg) * p.hkv + h;
                    bulk_g2s(sb + pp * geo.kc, p.k_codes + ph * geo.kc, geo.kc, &sh.full[s]);
                    bulk_g2s(sb + 2 * geo.kc + pp * geo.km,
                             reinterpret_cast<const uint8_t*>(p.k_meta) + ph * geo.km, geo.km, &sh.full[s]);
                    bulk_g2s(sb + 2 * (geo.kc + geo.km) + pp * geo.vc, p.v_codes + ph * geo.vc, geo.vc,
                             &sh.full[s]);
                    bulk_g2s(sb + 2 * (geo.kc + geo.km + geo.vc) + pp * geo.vm,
                             reinterpret_cast<const uint8_t*>(p.v_meta) + ph * geo.vm, geo.vm, &sh.full[s]);
                }
            }
        }
    } else if (warp == 13) {
        // ============================================================== MMA
        // the whole warp runs this loop with uniform values; one elected lane
        // issues each tcgen05 instruction
        const uint32_t qb_s = smem_u32(qb), pb_s = smem_u32(pb);
        const uint32_t cs_q = geo.cs_q;
        for (int i = 0; i <= ntot; ++i) {
            if (i < ntot) {
                const int u = i & 1;
                wait(&sh.kfull[u], (i >> 1) & 1);
                if (i >= 2) wait(&sh.sfree[u], ((i - 2) >> 1) & 1);
                if (__any_sync(FULL, !ok)) break;
                tc_fence_after();
                const uint64_t qd = smem_desc(qb_s + ((need_unrot && i >= ntiles) ? 16 * cs_q : 0u), cs_q, 128);
                const uint32_t dcol = tbase + COL_S + NS * u;
                const uint32_t acol = tbase + COL_AK + 64 * u;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc_mma_ts_warp(dcol, acol + 8 * k, qd + uint64_t((k * 2 * cs_q) >> 4), IDESC_S, k > 0 ? 1u : 0u);
                tc_commit_warp(&sh.kfree[u]);
                tc_commit_warp(&sh.sfull[u]);
            }
            if (i >= 1) {                                          // ·V MMA of tile i-1
                const int j = i - 1, u = j & 1;
                wait(&sh.vfull[u], (j >> 1) & 1);
                wait(&sh.pfull[u], (j >> 1) & 1);
                if (__any_sync(FULL, !ok)) break;
                tc_fence_after();
                const uint64_t pd = smem_desc(pb_s + u * 16 * CS_P, CS_P, 128);
                const uint32_t acol = tbase + COL_AV + 64 * u;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc_mma_ts_warp(tbase + COL_O, acol + 8 * k, pd + uint64_t((k * 2 * CS_P) >> 4), IDESC_O,
                                   (j > 0 || k > 0) ? 1u : 0u);
                tc_commit_warp(&sh.vfree[u]);
                tc_commit_warp(&sh.pfree[u]);
            }
        }
    } else if (warp < 4) {
        // ============================================================== keys
        const int pp_t = tid >> 6, slot_t = tid & 63;             // token t = tid
        for (int i = 0; i < ntot; ++i) {
            const int u = i & 1;
            const bool quant = i < ntiles;
            if (quant) wait(&sh.full[i % nst], (i / nst) & 1);
            if (i >= 2) wait(&sh.kfree[u], ((i - 2) >> 1) & 1);
            if (__any_sync(FULL, !ok)) break;                     // warp-uniform exit
            tc_fence_after();
            if (quant) {
                const uint8_t* kr = st + (i % nst) * geo.stage + pp_t * geo.kc + slot_t * 16;
#pragma unroll
                for (int c = 0; c < KW / 4; ++c) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(kr + c * (kPage * 16));
                    uint32_t a[4 * KREG];
                    Unpack<KB>::word(w4.x, &a[0 * KREG]);
                    Unpack<KB>::word(w4.y, &a[1 * KREG]);
                    Unpack<KB>::word(w4.z, &a[2 * KREG]);
                    Unpack<KB>::word(w4.w, &a[3 * KREG]);
                    tmem_st<4 * KREG>(tbase + lane_off + COL_AK + 64 * u + c * 4 * KREG, a);
                }
            } else {
                // bf16 window key of token t, permuted into the operand's channel order
                const bool valid = Lq + (i - ntiles) * 128 + tid < L;
                int slot = wslot0 + (i - ntiles) * 128 + tid;
                slot = valid ? (slot >= p.W ? slot - p.W : slot) : 0;
                const uint4* kr = reinterpret_cast<const uint4*>(p.k_win + ((size_t(b) * p.hkv + h) * p.W + slot) * D);
#pragma unroll
                for (int c = 0; c < 4; ++c) {                  // 32 channels -> 16 registers
                    uint32_t wv[16];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint4 w4 = valid ? kr[c * 4 + k] : make_uint4(0, 0, 0, 0);
                        wv[4 * k + 0] = w4.x; wv[4 * k + 1] = w4.y; wv[4 * k + 2] = w4.z; wv[4 * k + 3] = w4.w;
                    }
                    uint32_t a[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        const int ja = elem_at(2 * (16 * c + r), KB) - 32 * c;
                        const int jb = elem_at(2 * (16 * c + r) + 1, KB) - 32 * c;
                        a[r] = __byte_perm(wv[ja >> 1], wv[jb >> 1],
                                           ((ja & 1) ? 0x32u : 0x10u) | ((jb & 1) ? 0x7600u : 0x5400u));
                    }
                    tmem_st<16>(tbase + lane_off + COL_AK + 64 * u + c * 16, a);
                }
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sh.kfull[u]);
                if (quant) mbar_arrive(&sh.empty[i % nst]);
            }
        }
    } else if (warp >= 8) {
        // ============================================================== values
        const int j = tid - 256;                                  // channel
        for (int i = 0; i < ntot; ++i) {
            const int u = i & 1;
            const bool quant = i < ntiles;
            if (quant) wait(&sh.full[i % nst], (i / nst) & 1);
            if (i >= 2) wait(&sh.vfree[u], ((i - 2) >> 1) & 1);
            if (__any_sync(FULL, !ok)) break;                     // warp-uniform exit
            tc_fence_after();
            if (quant) {
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    const uint8_t* vb0 = st + (i % nst) * geo.stage + 2 * (geo.kc + geo.km) + pp * geo.vc;
                    if constexpr (VB == 1) {                     // one 8-byte chunk per channel
                        const uint2 w2 = *reinterpret_cast<const uint2*>(vb0 + j * 8);
                        uint32_t a[2 * VREG];
                        Unpack<VB>::word(w2.x, &a[0]);
                        Unpack<VB>::word(w2.y, &a[VREG]);
                        tmem_st<2 * VREG>(tbase + lane_off + COL_AV + 64 * u + pp * 32, a);
                    } else {                                     // VWP/4 chunks of 16 bytes, chunk-major
#pragma unroll
                        for (int c = 0; c < VWP / 4; ++c) {
                            const uint4 w4 = *reinterpret_cast<const uint4*>(vb0 + c * (D * 16) + j * 16);
                            uint32_t a[4 * VREG];
                            Unpack<VB>::word(w4.x, &a[0 * VREG]);
                            Unpack<VB>::word(w4.y, &a[1 * VREG]);
                            Unpack<VB>::word(w4.z, &a[2 * VREG]);
                            Unpack<VB>::word(w4.w, &a[3 * VREG]);
                            tmem_st<4 * VREG>(tbase + lane_off + COL_AV + 64 * u + pp * 32 + c * 4 * VREG, a);
                        }
                    }
                }
            } else {
                // bf16 window values of channel j, in the operand's token order
                const int base = (i - ntiles) * 128;
                const int nval = min(128, L - Lq - base);
                const __nv_bfloat16* vcol = p.v_win + (size_t(b) * p.hkv + h) * size_t(p.W) * D + j;
#pragma unroll
                for (int c = 0; c < 4; ++c) {                      // 32 tokens -> 16 registers
                    uint16_t vv[32];
#pragma unroll
                    for (int r = 0; r < 32; ++r) {                 // all loads first
                        const int kp = 32 * c + r;
                        const int t = (kp >> 6) * kPage + elem_at(kp & 63, VB);
                        int sl = wslot0 + base + t;
                        sl = sl >= p.W ? sl - p.W : sl;
                        vv[r] = t < nval ? __bfloat16_as_ushort(vcol[size_t(sl) * D]) : (uint16_t)0;
                    }
                    uint32_t a[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) a[r] = uint32_t(vv[2 * r]) | (uint32_t(vv[2 * r + 1]) << 16);
                    tmem_st<16>(tbase + lane_off + COL_AV + 64 * u + c * 16, a);
                }
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sh.vfull[u]);
                if (quant) mbar_arrive(&sh.empty[i % nst]);
            }
        }
    } else {
        // ============================================================== softmax
        const int t = tid - 128;                                  // token
        const int sw = warp - 4;                                  // softmax warp 0..3
        const int pp_t = t >> 6, slot_t = t & 63;
        const int kpos_t = pp_t * kPage + kpos_of(slot_t, VB);    // position along the ·V K dim
        float mrun[NH], lpart[NH], pzpart[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            mrun[r] = -INFINITY;
            lpart[r] = 0.0f;
            pzpart[r] = 0.0f;
        }
        for (int i = 0; i < ntot; ++i) {
            const int u = i & 1;
            const bool quant = i < ntiles;
            bool valid;
            float ksc[kKGroups], kzp[kKGroups], vsc = 0.0f, vzp = 0.0f;
            if (quant) {
                wait(&sh.full[i % nst], (i / nst) & 1);
                const uint8_t* sb = st + (i % nst) * geo.stage;
                const int lp = pg0 + 2 * i + pp_t;
                valid = lp < pg1 && lp * kPage + slot_t < Lq && sh.pages[2 * i + pp_t] >= 0;
                const uint4 m4 = *reinterpret_cast<const uint4*>(sb + 2 * geo.kc + pp_t * geo.km + slot_t * 16);
                const uint32_t mw[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                for (int grp = 0; grp < kKGroups; ++grp) {
                    const float2 f = meta_f2(mw[grp]);
                    ksc[grp] = f.x;
                    kzp[grp] = f.y;
                }
                if (valid) {
                    const float2 f = meta_f2(*reinterpret_cast<const uint32_t*>(
                        sb + 2 * (geo.kc + geo.km + geo.vc) + pp_t * geo.vm + slot_t * 4));
                    vsc = f.x;
                    vzp = f.y;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.empty[i % nst]);
            } else {
                valid = Lq + (i - ntiles) * 128 + t < L;
#pragma unroll
                for (int grp = 0; grp < kKGroups; ++grp) {
                    ksc[grp] = 1.0f;
                    kzp[grp] = 0.0f;
                }
                vsc = valid ? 1.0f : 0.0f;
            }
            // ---- scores of token t
            wait(&sh.sfull[u], (i >> 1) & 1);
            tc_fence_after();
            uint32_t ds[NS];
#pragma unroll
            for (int c = 0; c < NS / 16; ++c)
                tmem_ld16(tbase + lane_off + COL_S + NS * u + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&ds[c * 16]));
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.sfree[u]);
            float sc[NH];
            bool exceed = false;
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                const float4 qs4 = sh.qsum[r < g ? r : 0];
                const float qs[4] = {qs4.x, qs4.y, qs4.z, qs4.w};
                float acc = 0.0f;
#pragma unroll
                for (int grp = 0; grp < kKGroups; ++grp) {
                    const float dot = __uint_as_float(ds[r * 8 + 2 * grp]) + __uint_as_float(ds[r * 8 + 2 * grp + 1]);
                    acc = fmaf(ksc[grp], dot, fmaf(kzp[grp], qs[grp], acc));
                }
                sc[r] = (valid && r < g) ? acc * scale_log2 : -INFINITY;
                exceed |= sc[r] > mrun[r] + kLazyMax;
            }
            // ---- running max shared by the 4 softmax warps
            // the vote also carries a failed wait, so the 4 warps leave together
            const int wv = (__any_sync(FULL, exceed) ? 1 : 0) | (__any_sync(FULL, !ok) ? 2 : 0);
            if (lane == 0) sh.vote[u][sw] = wv;
            named_sync(1, 128);
            const int votes = sh.vote[u][0] | sh.vote[u][1] | sh.vote[u][2] | sh.vote[u][3];
            if (votes & 2) {
                ok = false;
                break;
            }
            if (votes & 1) {
                // exact max of the tile; rescale the sums and the ·V accumulator
#pragma unroll
                for (int r = 0; r < NH; ++r) {
                    const float m = warp_max(sc[r]);
                    if (lane == 0) reinterpret_cast<float*>(&sh.red[u][r])[sw] = m;
                }
                named_sync(1, 128);
                float alpha[NH];
#pragma unroll
                for (int r = 0; r < NH; ++r) {
                    const float4 rv = sh.red[u][r];
                    const float mnew = fmaxf(mrun[r], fmaxf(fmaxf(rv.x, rv.y), fmaxf(rv.z, rv.w)));
                    const float mu = (mnew == -INFINITY) ? 0.0f : mnew;
                    alpha[r] = ex2(mrun[r] - mu);
                    lpart[r] *= alpha[r];
                    pzpart[r] *= alpha[r];
                    mrun[r] = mnew;
                }
                if (i >= 1) {
                    wait(&sh.pfree[(i - 1) & 1], ((i - 1) >> 1) & 1);       // ·V MMA of tile i-1 done
                    tc_fence_after();
                    uint32_t o[16];
                    tmem_ld16(tbase + lane_off + COL_O, o);
                    tc_wait_ld();
#pragma unroll
                    for (int n = 0; n < 16; ++n)
                        o[n] = __float_as_uint(__uint_as_float(o[n]) * alpha[(n >> 1) < NH ? (n >> 1) : 0]);
                    tmem_st16(tbase + lane_off + COL_O, o);
                    tc_wait_st();
                }
            }
            // ---- P' of token t into buffer u (free once the ·V MMA of tile i-2 is done)
            if (i >= 2) wait(&sh.pfree[u], ((i - 2) >> 1) & 1);
            uint8_t* pbu = pb + u * 16 * CS_P;
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                if (r >= g) continue;
                const float mu = (mrun[r] == -INFINITY) ? 0.0f : mrun[r];
                const float pr = ex2(sc[r] - mu);
                lpart[r] += pr;
                pzpart[r] = fmaf(pr, vzp, pzpart[r]);
                const float pv = pr * vsc;
                const float hi = __bfloat162float(__float2bfloat16_rn(pv));
                *reinterpret_cast<uint16_t*>(pbu + b_off(2 * r, kpos_t, CS_P)) = bf16_bits(pv);
                *reinterpret_cast<uint16_t*>(pbu + b_off(2 * r + 1, kpos_t, CS_P)) = bf16_bits(pv - hi);
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.pfull[u]);
        }
        // ---- partial of this split: o for channel 32*sw + lane, m, l
        const int last_i = ntot - 1;
        wait(&sh.pfree[last_i & 1], (last_i >> 1) & 1);
        tc_fence_after();
        uint32_t o[16];
        tmem_ld16(tbase + lane_off + COL_O, o);
        tc_wait_ld();
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            const float l = warp_sum(lpart[r]);
            const float z = warp_sum(pzpart[r]);
            if (lane == 0) {
                reinterpret_cast<float*>(&sh.red[0][r])[sw] = l;
                reinterpret_cast<float*>(&sh.red2[r])[sw] = z;
            }
        }
        named_sync(1, 128);
        const bool bad = !ok || sh.abort;
        const int ch = 32 * sw + lane;
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            if (r >= g) continue;
            const float4 zv = sh.red2[r];
            const float z = (zv.x + zv.y) + (zv.z + zv.w);
            const float val = __uint_as_float(o[2 * r]) + __uint_as_float(o[2 * r + 1]) + z;
            ws_o[(row0 + size_t(r) * slots + split) * D + ch] = bad ? NAN : val;
            if (t == 0) {
                const float4 lv = sh.red[0][r];
                const float l = (lv.x + lv.y) + (lv.z + lv.w);
                ws_ml[(row0 + size_t(r) * slots + split) * 2 + 0] = bad ? 0.0f : mrun[r];
                ws_ml[(row0 + size_t(r) * slots + split) * 2 + 1] = bad ? NAN : l;
            }
        }
        if (bad && t == 0) atomicAdd(&g_tc_wait_timeouts, 1u);
    }
    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (sh.abort && tid == 0) {
        // let copies still in flight land before the shared memory is released
        for (int s = 0; s < nst; ++s) mbar_wait(&sh.full[s], 0, kWaitNs / 16);
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

template <int KB, int VB, int NS>
cudaError_t launch_tc_t(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                        float scale_log2, float* ws_o, float* ws_ml, const DecodePlan& pl, cudaStream_t s) {
    const TcGeom geo = tc_geom(p, NS, 227 * 1024);
    if (geo.nstages < 2) return cudaErrorNotSupported;
    auto kern = decode_tc_kernel<KB, VB, NS>;
    static int configured = 0;
    if (configured < geo.total) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.total);
        if (e != cudaSuccess) return e;
        configured = geo.total;
    }
    dim3 grid(pl.grid_x, p.hkv, p.batch);
    kern<<<grid, kThreads, geo.total, s>>>(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl.pages_per_split,
                                          pl.total_splits, geo);
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

// one CTA per SM (it holds all 512 tensor-memory columns)
int tc_ctas_per_sm(const Params& p) { return 1; }

cudaError_t launch_decode_tc(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                             float scale_log2, float* ws_o, float* ws_ml, const DecodePlan& pl, cudaStream_t s) {
    if (p.g <= 4) return dispatch_bits<32>(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl, s);
    return dispatch_bits<64>(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl, s);
}

}  // namespace kvq

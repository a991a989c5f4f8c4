// Decode attention over the quantized cache on the 5th-generation tensor
// cores (tcgen05, sm_100a): head_dim 128, key groups of 32 channels, value
// groups of 128 channels, any key/value bit widths in {1, 2, 4, 8}.
//
// Attention ("Kuantisasi KV cache mengganggu attention ...", section "Error
// pada key masuk sebelum softmax"): s = q K^T * sm_scale, a = softmax(s),
// o = a V, with dequantization fused into the kernel (section "Pertumbuhan
// cache mengubah trade pada serving").  With x^ = c*scale + zero per group:
//   q . k^ = sum_groups ( scale * (q . c)_group + zero * (sum q)_group )
//   o      = sum_t (p_t scale_t) c_t + sum_t p_t zero_t
// Both contractions run on the tensor cores over the raw integer codes:
//  - scores: kind::i8.  Key codes are exact int8 (8-bit codes offset by
//    -128, folded into the zero point); the fp32 query of each head is split
//    into three int8 limbs a + b/2^7 + c/2^14 times a power of two (exact to
//    2^-20 of the head's largest element), one column per (head, key group,
//    limb) so that the group scales apply after the product;
//  - values: kind::f16.  Value codes are exact bf16; P' = p * value_scale is
//    a bf16 pair (high part + remainder), accumulated in fp32 in tensor
//    memory across the whole split.
//
// One CTA per (sequence, kv-head, split of at most 16 tiles of 128 tokens),
// 288 threads, two CTAs per SM when they fit.  Two phases:
//   1. scores: loader warps unpack key codes to int8 in tensor memory
//      (double buffered), the MMA warp multiplies them with the query limbs,
//      the softmax warps turn the s32 products into fp32 scores, keep them in
//      shared memory and track their maximum;
//   2. values: with the exact maximum known, the softmax warps write
//      P' = 2^(s - max) * value_scale as a bf16 pair, the loader warps unpack
//      value codes to bf16 in tensor memory (double buffered in the columns
//      phase 1 used), and the MMA warp accumulates ·V in tensor memory.
// Warps 0-3 softmax (thread t owns token t of each tile: metadata, scores,
// P'), warps 4-7 loaders (thread i owns token i's key codes and channel i's
// value codes; per-thread cp.async into a ring of shared-memory stages that
// runs through both phases), warp 8 issues every MMA (one elected lane).
// Hand-overs go through mbarriers; every wait is bounded.  The bf16 window
// positions are handled by separate CTAs of the same grid on CUDA cores
// (fp32), each writing its own partial.
#pragma once

#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_tc_ptx.cuh"

namespace kvq {
namespace tc {

using namespace ptx;

constexpr int D = 128;
constexpr int TILE = 128;                     // tokens per tile (two pages)
constexpr int NKG = 4;                        // key groups of 32 channels
constexpr int kThreads = 288;
constexpr int kMaxPagesPerSplit = 256;
constexpr int kMaxTiles = 16;                 // tiles per quantized split (scores are kept in shared memory)
constexpr int kWinPerSplit = kTcWindowPerCta;   // window positions per window CTA (one chunk)
constexpr int WCH = 64;                       // window positions per chunk
constexpr int kWinSmem = 2 * WCH * D * 2;     // key and value rows of a chunk
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr unsigned FULL = 0xffffffffu;


constexpr int ns_cols(int nhc) { return ((12 * nhc + 15) / 16) * 16; }
// score accumulator buffers: two when they fit in 256 columns with the rest
constexpr int s_bufs(int nhc) { return 64 + 2 * ns_cols(nhc) + 16 <= 256 ? 2 : 1; }

template <int KB, int VB, int NHC>
struct Cfg {
    static constexpr int NS = ns_cols(NHC);                  // score columns (head, key group, limb)
    static constexpr int SB = s_bufs(NHC);                   // score accumulator buffers
    static constexpr int NO = 16;                            // ·V columns (head, high / remainder)
    // tensor-memory columns.  Phase 1: key operands (int8) at 0 and 32, score
    // accumulators from 64.  Phase 2: value operands (bf16) at 0 and 64,
    // over the phase-1 columns.  The ·V accumulator after both.
    static constexpr int COL_AK = 0;
    static constexpr int COL_S = 64;
    static constexpr int COL_AV = 0;
    static constexpr int COL_O = COL_S + SB * NS;
    static constexpr int TMEM_COLS = 256;
    static_assert(COL_S + SB * NS >= 128, "second value operand lies inside the phase-1 columns");
    static_assert(COL_O + NO <= TMEM_COLS, "tensor-memory plan fits 256 columns");
    static constexpr int KROW = D * KB / 8;                  // key row bytes of one token
    static constexpr int VCH = kPage * VB / 8;               // value bytes of one channel in one page
    // one ring stage holds either a key step (codes [chunk][token][16 B],
    // key meta [token][16 B]) or a value step (codes [chunk][channel][16 B],
    // value meta in the first 4 bytes of [token][16 B]).  Every thread reads
    // back only bytes it copied itself, in both phases: warps run at their
    // own pace, so no two threads may share bytes of a stage.
    static constexpr int CODES = TILE * KROW > D * 2 * VCH ? TILE * KROW : D * 2 * VCH;
    static constexpr int ST_M = CODES;
    static constexpr int STAGE = CODES + TILE * 16;
    static constexpr int CS_Q = NS * 16 + 16;                // chunk stride of the query operand
    static constexpr int CS_P = 16 * 16 + 16;                // chunk stride of the P' operand
    static_assert(2 * NHC <= NO, "two ·V columns per head");
};

struct Shared {
    uint64_t kfull[2];       // loaders -> MMA: key operand written
    uint64_t sfull[2];       // MMA -> softmax, loaders: score products ready (key operand read)
    uint64_t sfree[2];       // softmax -> MMA, loaders: score accumulator read
    uint64_t vfull[2];       // loaders -> MMA: value operand written
    uint64_t pfull[2];       // softmax -> MMA: P' operand written
    uint64_t pvdone[2];      // MMA -> softmax, loaders: ·V product of the tile done
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
    float smax[4][kMaxGqa];              // softmax warps: score maxima
    float red[4][kMaxGqa], red2[4][kMaxGqa];
    alignas(16) float qsum[kMaxGqa][NKG];   // sums of the rotated query per key group
    float qs0[kMaxGqa];                  // query limb unit: 2^-14 of the head's s0
    alignas(16) float qf[kMaxGqa][D];    // query, fp32, as given
    alignas(16) float qr[kMaxGqa][D];    // query rotated like the stored keys
    alignas(16) float wsc[kMaxGqa][TILE];   // window CTAs: scores / weights of a chunk
    float wred[8][kMaxGqa];
    int pages[kMaxPagesPerSplit];
};

// Shared-memory plan: Shared, the query operand, two P' buffers, the scores
// of the split, then a ring of R stages.  Two CTAs share an SM when three
// stages still fit in half the shared memory; otherwise one.
constexpr int stage_bytes(int kb, int vb) {
    return (TILE * (D * kb / 8) > D * 2 * (kPage * vb / 8) ? TILE * (D * kb / 8) : D * 2 * (kPage * vb / 8)) +
           TILE * 16;
}
constexpr int ring_offset(int nhc) {
    return ((((int(sizeof(Shared)) + 127) & ~127) + 8 * (ns_cols(nhc) * 16 + 16) + 2 * 16 * (16 * 16 + 16) +
             kMaxTiles * nhc * TILE * 4) + 127) & ~127;
}
constexpr int ctas_per_sm(int kb, int vb, int nhc) {
    return (112 * 1024 - ring_offset(nhc)) / stage_bytes(kb, vb) >= 3 ? 2 : 1;
}

template <int KB, int VB, int NHC>
struct Layout {
    using C = Cfg<KB, VB, NHC>;
    static constexpr int CTAS = ctas_per_sm(KB, VB, NHC);
    static constexpr int OFF_QB = (int(sizeof(Shared)) + 127) & ~127;
    static constexpr int OFF_PB = OFF_QB + 8 * C::CS_Q;
    static constexpr int OFF_SC = OFF_PB + 2 * 16 * C::CS_P;          // scores [tile][head][token] fp32
    static constexpr int OFF_RING = (OFF_SC + kMaxTiles * NHC * TILE * 4 + 127) & ~127;
    static constexpr int BUDGET = CTAS == 2 ? 112 * 1024 : 224 * 1024;
    static constexpr int R0 = (BUDGET - OFF_RING) / C::STAGE;
    static constexpr int R = R0 > 8 ? 8 : R0;                 // ring stages
    static constexpr int USED = OFF_RING + R * C::STAGE;
    // never more CTAs per SM than planned (the tensor memory holds no more)
    static constexpr int MIN_TOTAL = CTAS == 2 ? 80 * 1024 : 120 * 1024;
    static constexpr int TOTAL = USED > MIN_TOTAL ? USED : MIN_TOTAL;
    static_assert(R >= 3, "ring needs three stages");
    static_assert(OFF_RING == ring_offset(NHC) && C::STAGE == stage_bytes(KB, VB), "plan formulas agree");
    static_assert(OFF_SC + kWinSmem <= TOTAL && 4 * D * kMaxGqa * 4 <= WCH * D * 2 * 2,
                  "window rows and the reduction buffer fit from the score area on");
};

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ float ex2(float x) {   // 2^x, hardware approximation (flushes subnormals)
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
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
__device__ __forceinline__ int rni(float x) {
    int r;
    asm("cvt.rni.s32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// cp.async: 16 / 8 / 4 bytes global -> shared; src_bytes 0 fills zeros
__device__ __forceinline__ void cp16(void* dst, const void* src, bool have) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(have ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp8(void* dst, const void* src, bool have) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(have ? 8 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp4(void* dst, const void* src, bool have) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(have ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// kind::i8 MMA, A from tensor memory, issued by one elected lane of a warp
__device__ __forceinline__ void mma_i8_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}
// instruction descriptor: signed int8 A and B (K-major), s32 accumulator
__host__ __device__ constexpr uint32_t idesc_s8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- unpacking
// A 32-bit word of b-bit codes -> 8/b words of int8 codes: word s holds, in
// byte k, the code of element k*(8/b) + s.  So K position 4*s + k of the
// word's run carries element k*(8/b) + s; 8-bit codes are offset by -128.
template <int B>
__device__ __forceinline__ void unpack_i8(uint32_t w, uint32_t* o) {
    if constexpr (B == 8) {
        o[0] = w ^ 0x80808080u;
    } else {
        constexpr uint32_t M = B == 4 ? 0x0F0F0F0Fu : B == 2 ? 0x03030303u : 0x01010101u;
#pragma unroll
        for (int s = 0; s < 8 / B; ++s) o[s] = (w >> (B * s)) & M;
    }
}
// K position (within a run of 32/b-element words) of element e
__host__ __device__ __forceinline__ int kpos_of(int e, int bits) {
    const int per = 32 / bits, f = 8 / bits;
    const int w = e / per, r = e % per;
    return w * per + 4 * (r % f) + r / f;
}
// byte offset of (row n, K position kp) in a K-major int8 B operand stored as
// [16-byte K chunk][row][16 bytes] with chunk stride cs
__device__ __forceinline__ int b_off(int n, int kp, int cs) { return (kp >> 4) * cs + n * 16 + (kp & 15); }

// the bf16 bits of a pair, as floats
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------- value codes -> bf16
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

// position (along the MMA K dimension) of element i of a packed run of value codes
__host__ __device__ __forceinline__ int kpos_bf16(int i, int bits) {
    const int per = 32 / bits, half = per / 2;
    const int w = i / per, r = i % per;
    return w * per + 2 * (r % half) + r / half;
}
// byte offset of element (row n, K position pos) in a K-major B operand
// stored as [k step][half][row][8 x bf16] with chunk stride cs
__device__ __forceinline__ int b_off_bf16(int n, int pos, int cs) {
    return ((pos >> 4) * 2 + ((pos >> 3) & 1)) * cs + n * 16 + (pos & 7) * 2;
}


__device__ __forceinline__ uint16_t bf16_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }


static __device__ void write_empty_partial(int g, float* ws_o, float* ws_ml, size_t row0, int slots, int slot) {
    for (int i = threadIdx.x; i < g * D; i += blockDim.x) {
        const int r = i / D;
        ws_o[(row0 + size_t(r) * slots + slot) * D + (i % D)] = 0.0f;
        if (i % D == 0) {
            ws_ml[(row0 + size_t(r) * slots + slot) * 2 + 0] = -INFINITY;
            ws_ml[(row0 + size_t(r) * slots + slot) * 2 + 1] = 0.0f;
        }
    }
}

// --------------------------------------------------------- window partial
// CUDA-core attention over window positions [w0, w1) (bf16 keys and values,
// unrotated query) in chunks of 64 positions with an online softmax.  Every
// thread of the CTA copies a share of the chunk's key and value rows into
// shared memory (cp.async); warps 0-7 then compute from shared memory:
//   scores:  four threads per position, 32 channels each;
//   ·V:      thread (jp, tq) owns channels 2jp, 2jp+1 and positions tq mod 4;
//            the four position classes are summed through shared memory.

template <int NHC>
__device__ __forceinline__ void window_partial(const Params& p, Shared& sh, uint8_t* buf, int b, int h, int w0,
                                               int w1, float scale_log2, float* ws_o, float* ws_ml, size_t row0,
                                               int slots, int slot) {
    const int g = p.g, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool cw = warp < 8;                  // compute warps
    const int t = (tid >> 2) & (WCH - 1), qq = tid & 3;   // scores: position t, channel quarter qq
    const int jp = tid & 63, tq = (tid >> 6) & 3;          // ·V: channel pair, position class
    const __nv_bfloat16* krow = reinterpret_cast<const __nv_bfloat16*>(buf);
    const __nv_bfloat16* vrow = reinterpret_cast<const __nv_bfloat16*>(buf + WCH * D * 2);
    float* scratch = reinterpret_cast<float*>(buf);         // reuses the key rows at the end
    float m[NHC], l[NHC], o0[NHC], o1[NHC];
#pragma unroll
    for (int r = 0; r < NHC; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.0f;
        o0[r] = 0.0f;
        o1[r] = 0.0f;
    }
    const size_t hb = (size_t(b) * p.hkv + h) * size_t(p.W);
    for (int c0 = w0; c0 < w1; c0 += WCH) {
        const int n = min(WCH, w1 - c0);
        // ---- rows of the chunk -> shared memory (16-byte pieces, keys then values)
        for (int idx = tid; idx < 2 * n * 16; idx += kThreads) {
            const int kv = idx >= n * 16, rem = kv ? idx - n * 16 : idx;
            const int row = rem >> 4, piece = rem & 15;
            const size_t src = (hb + size_t((c0 + row) % p.W)) * D + piece * 8;
            cp16(buf + kv * (WCH * D * 2) + row * (D * 2) + piece * 16, (kv ? p.v_win : p.k_win) + src, true);
        }
        cp_commit();
        cp_wait<0>();
        __syncthreads();
        float s[NHC];
#pragma unroll
        for (int r = 0; r < NHC; ++r) s[r] = -INFINITY;
        if (cw) {
            // ---- scores: thread (t, qq) takes channels 32qq .. 32qq+31 of position t
            float acc[NHC];
#pragma unroll
            for (int r = 0; r < NHC; ++r) acc[r] = 0.0f;
            const bool in = t < n;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int cc = (c + (t >> 1)) & 3;             // rotate the 16-byte pieces across lanes
                const uint4 w4 = in ? *reinterpret_cast<const uint4*>(krow + t * D + 32 * qq + 8 * cc)
                                    : make_uint4(0, 0, 0, 0);
                const float kv[8] = {bf_lo(w4.x), bf_hi(w4.x), bf_lo(w4.y), bf_hi(w4.y),
                                     bf_lo(w4.z), bf_hi(w4.z), bf_lo(w4.w), bf_hi(w4.w)};
#pragma unroll
                for (int r = 0; r < NHC; ++r) {
                    if (r < g) {
                        const float4 qa = *reinterpret_cast<const float4*>(&sh.qf[r][32 * qq + 8 * cc]);
                        const float4 qb = *reinterpret_cast<const float4*>(&sh.qf[r][32 * qq + 8 * cc + 4]);
                        acc[r] = fmaf(qa.x, kv[0], acc[r]);
                        acc[r] = fmaf(qa.y, kv[1], acc[r]);
                        acc[r] = fmaf(qa.z, kv[2], acc[r]);
                        acc[r] = fmaf(qa.w, kv[3], acc[r]);
                        acc[r] = fmaf(qb.x, kv[4], acc[r]);
                        acc[r] = fmaf(qb.y, kv[5], acc[r]);
                        acc[r] = fmaf(qb.z, kv[6], acc[r]);
                        acc[r] = fmaf(qb.w, kv[7], acc[r]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < NHC; ++r) {
                float tot = acc[r] + __shfl_xor_sync(FULL, acc[r], 1);
                tot += __shfl_xor_sync(FULL, tot, 2);
                s[r] = (in && r < g) ? tot * scale_log2 : -INFINITY;
                const float wm = warp_max(s[r]);
                if (lane == 0 && r < g) sh.wred[warp][r] = wm;
            }
        }
        __syncthreads();
        if (cw) {
#pragma unroll
            for (int r = 0; r < NHC; ++r) {
                if (r < g) {
                    float cm = sh.wred[0][r];
#pragma unroll
                    for (int w = 1; w < 8; ++w) cm = fmaxf(cm, sh.wred[w][r]);
                    const float mnew = fmaxf(m[r], cm);
                    const float alpha = (mnew == -INFINITY) ? 1.0f : ex2(m[r] - mnew);
                    m[r] = mnew;
                    const float pr = (s[r] == -INFINITY) ? 0.0f : ex2(s[r] - mnew);
                    l[r] = fmaf(l[r], alpha, qq == 0 ? pr : 0.0f);
                    if (qq == 0) sh.wsc[r][t] = pr;
                    o0[r] *= alpha;
                    o1[r] *= alpha;
                }
            }
        }
        __syncthreads();
        if (cw) {
            // ---- ·V: positions tq, tq+4, ... of the chunk, channels 2jp, 2jp+1
#pragma unroll 4
            for (int k = 0; k < WCH / 4; ++k) {
                const int tt = tq + 4 * k;
                if (tt < n) {
                    const uint32_t vv = *reinterpret_cast<const uint32_t*>(vrow + tt * D + 2 * jp);
                    const float va = bf_lo(vv), vb = bf_hi(vv);
#pragma unroll
                    for (int r = 0; r < NHC; ++r) {
                        if (r < g) {
                            const float pr = sh.wsc[r][tt];
                            o0[r] = fmaf(pr, va, o0[r]);
                            o1[r] = fmaf(pr, vb, o1[r]);
                        }
                    }
                }
            }
        }
        __syncthreads();                            // rows, wsc and wred are rewritten next
    }
    // position classes -> channel sums; l over the score threads
    if (cw) {
#pragma unroll
        for (int r = 0; r < NHC; ++r) {
            if (r < g) {
                scratch[(tq * kMaxGqa + r) * D + 2 * jp] = o0[r];
                scratch[(tq * kMaxGqa + r) * D + 2 * jp + 1] = o1[r];
            }
            const float ls = warp_sum(l[r]);
            if (lane == 0 && r < g) sh.wred[warp][r] = ls;
        }
    }
    __syncthreads();
    if (tid < D) {
        const int j = tid;
#pragma unroll
        for (int r = 0; r < NHC; ++r) {
            if (r >= g) continue;
            const float v = (scratch[(0 * kMaxGqa + r) * D + j] + scratch[(1 * kMaxGqa + r) * D + j]) +
                            (scratch[(2 * kMaxGqa + r) * D + j] + scratch[(3 * kMaxGqa + r) * D + j]);
            const size_t row = row0 + size_t(r) * slots + slot;
            ws_o[row * D + j] = v;
            if (j == 0) {
                float ls = 0.0f;
#pragma unroll
                for (int w = 0; w < 8; ++w) ls += sh.wred[w][r];
                ws_ml[row * 2 + 0] = m[r];
                ws_ml[row * 2 + 1] = ls;
            }
        }
    }
}

// ------------------------------------------------------------------ kernel
// grid (Hkv, B, splits_q + nws); the block scheduler dispatches in linear
// order, so the split index is the slowest dimension.  z < splits_q:
// quantized split z covering pages [z*pps, (z+1)*pps); the nws window CTAs
// come last and cover window positions [Lq + w*64, Lq + (w+1)*64).  Every
// CTA writes one partial (m, l, o) per query head into slot z.
template <int KB, int VB, int NHC>
__global__ void __launch_bounds__(kThreads, ctas_per_sm(KB, VB, NHC))
decode_tc_kernel(const Params p, const void* __restrict__ q, const int q_bf16, const int32_t* __restrict__ lens,
                 const int max_len, const float scale_log2, float* __restrict__ ws_o, float* __restrict__ ws_ml,
                 const int pps, const int nws, const int slots, unsigned int* __restrict__ status) {
    using C = Cfg<KB, VB, NHC>;
    using LY = Layout<KB, VB, NHC>;
    constexpr int R = LY::R;
    constexpr int NS = C::NS, SB = C::SB;
    constexpr uint32_t IDESC_S = idesc_s8(128, NS);
    constexpr uint32_t IDESC_O = idesc_bf16_f32(128, C::NO);
    constexpr int VWP = kPage * VB / 32;     // value words per channel per page
    constexpr int VREG = 16 / VB;            // bf16x2 registers per value word

    extern __shared__ __align__(1024) uint8_t smem[];
    Shared& sh = *reinterpret_cast<Shared*>(smem);
    uint8_t* qb = smem + LY::OFF_QB;
    uint8_t* pb = smem + LY::OFF_PB;
    uint8_t* ring = smem + LY::OFF_RING;
    float* scs = reinterpret_cast<float*>(smem + LY::OFF_SC);   // [tile][head][token]

    const int h = blockIdx.x, b = blockIdx.y, x = blockIdx.z;   // split index outermost: dispatched last
    const int g = p.g, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = max(0, min(lens[b], max_len));
    const int Lq = max(0, L - p.W);
    const size_t row0 = (size_t(b) * p.hq + size_t(h) * g) * slots;

    // ---- which work this CTA has
    // quantized splits first, so that they all start in the first wave of
    // CTAs; the short window CTAs fill the remaining slots and the tail
    const int nsq = (int)gridDim.z - nws;
    const bool is_win = x >= nsq;
    int w0 = 0, w1 = 0, pg0 = 0, pg1 = 0, ntiles = 0;
    if (is_win) {
        w0 = Lq + (x - nsq) * kWinPerSplit;
        w1 = min(L, w0 + kWinPerSplit);
    } else {
        const int npg = (Lq + kPage - 1) / kPage;
        pg0 = x * pps;
        pg1 = min(npg, pg0 + pps);
        ntiles = pg1 > pg0 ? (pg1 - pg0 + 1) / 2 : 0;
    }
    if ((is_win && w0 >= w1) || (!is_win && ntiles == 0)) {
        write_empty_partial(g, ws_o, ws_ml, row0, slots, x);
        return;
    }

    // ---- query (fp32; rotated copy for the quantized keys)
    for (int i = tid; i < g * D; i += kThreads) {
        const size_t off = (size_t(b) * p.hq + size_t(h) * g + i / D) * D + (i % D);
        sh.qf[i / D][i % D] = q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[off])
                                     : reinterpret_cast<const float*>(q)[off];
    }
    __syncthreads();
    if (is_win) {
        window_partial<NHC>(p, sh, smem + LY::OFF_SC, b, h, w0, w1, scale_log2, ws_o, ws_ml, row0, slots, x);
        return;
    }

    if (tid == 0) {
        for (int u = 0; u < 2; ++u) {
            mbar_init(&sh.kfull[u], 4);
            mbar_init(&sh.sfull[u], 1);
            mbar_init(&sh.sfree[u], 4);
            mbar_init(&sh.vfull[u], 4);
            mbar_init(&sh.pfull[u], 4);
            mbar_init(&sh.pvdone[u], 1);
        }
        mbar_init(&sh.mma_done, 1);
        mbar_fence_init();
        sh.abort = 0;
    }
    if (warp == 8) {
        tmem_alloc(&sh.tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    for (int i = tid; i < pg1 - pg0; i += kThreads) sh.pages[i] = phys_page(p, b, pg0 + i);
    for (int i = tid; i < 8 * C::CS_Q / 4; i += kThreads) reinterpret_cast<uint32_t*>(qb)[i] = 0u;
    for (int i = tid; i < 2 * 16 * C::CS_P / 4; i += kThreads) reinterpret_cast<uint32_t*>(pb)[i] = 0u;
    __syncthreads();
    // query operand: row n = 12r + 3grp + l (head r, key group grp, limb l),
    // K position of channel j in the int8 key operand; zeros outside the group.
    // One warp per head; lane owns channels 4*lane .. 4*lane+3.
    for (int r = warp; r < g; r += kThreads / 32) {
        float xr[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) xr[c] = sh.qf[r][lane * 4 + c];
        if (p.rotate) rotate_warp<D>(xr, p.signs, lane);
        float amax = fmaxf(fmaxf(fabsf(xr[0]), fabsf(xr[1])), fmaxf(fabsf(xr[2]), fabsf(xr[3])));
        amax = warp_max(amax);
        float gs = (xr[0] + xr[1]) + (xr[2] + xr[3]);
        gs += __shfl_xor_sync(FULL, gs, 1);
        gs += __shfl_xor_sync(FULL, gs, 2);
        gs += __shfl_xor_sync(FULL, gs, 4);                   // lanes 8grp .. 8grp+7 = key group grp
        if ((lane & 7) == 0) sh.qsum[r][lane >> 3] = gs;
        const uint32_t eb = __float_as_uint(amax) >> 23;      // biased exponent: amax < 2^(eb-126)
        const bool use = eb >= 40;
        const float inv_s0 = use ? __uint_as_float((259u - eb) << 23) : 0.0f;   // 2^(132-eb) = 1/s0
        if (lane == 0) sh.qs0[r] = use ? __uint_as_float((eb - 19u) << 23) : 0.0f;   // s0 * 2^-14
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int j = lane * 4 + c, grp = j >> 5, kp = kpos_of(j, KB);
            const float xs = xr[c] * inv_s0;                   // |xs| < 64, exact
            const int a = rni(xs);
            const float r1 = (xs - (float)a) * 128.0f;
            const int bl = rni(r1);
            const float r2 = (r1 - (float)bl) * 128.0f;
            const int cl = rni(r2);
            const int n0 = 12 * r + 3 * grp;
            qb[b_off(n0 + 0, kp, C::CS_Q)] = (uint8_t)(int8_t)a;
            qb[b_off(n0 + 1, kp, C::CS_Q)] = (uint8_t)(int8_t)bl;
            qb[b_off(n0 + 2, kp, C::CS_Q)] = (uint8_t)(int8_t)cl;
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sh.tmem_base;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;     // this warp's tensor-memory lanes
    const int nt = ntiles;
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
    // ring steps: step k < nt is key tile k, step k >= nt is value tile k - nt

    if (warp == 8) {
        // =============================================================== MMA
        const uint64_t qd = smem_desc(smem_u32(qb), C::CS_Q, 128);
        for (int i = 0; i < nt; ++i) {                         // phase 1: scores
            const int sb = i % SB;
            wait(&sh.kfull[i & 1], (i >> 1) & 1);
            if (i >= SB) wait(&sh.sfree[sb], ((i - SB) / SB) & 1);   // softmax read the accumulator
            if (__any_sync(FULL, !ok)) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_i8_warp(tbase + C::COL_S + NS * sb, tbase + C::COL_AK + 32 * (i & 1) + 8 * k,
                            qd + uint64_t((k * 2 * C::CS_Q) >> 4), IDESC_S, k > 0 ? 1u : 0u);
            tc_commit_warp(&sh.sfull[sb]);
        }
        ok = __all_sync(FULL, ok);
        const uint32_t pb_s = smem_u32(pb);
        for (int j = 0; j < nt && ok; ++j) {                   // phase 2: ·V
            const int u = j & 1;
            wait(&sh.vfull[u], (j >> 1) & 1);
            wait(&sh.pfull[u], (j >> 1) & 1);
            if (__any_sync(FULL, !ok)) break;
            tc_fence_after();
            const uint64_t pd = smem_desc(pb_s + u * 16 * C::CS_P, C::CS_P, 128);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                tc_mma_ts_warp(tbase + C::COL_O, tbase + C::COL_AV + 64 * u + 8 * k,
                               pd + uint64_t((k * 2 * C::CS_P) >> 4), IDESC_O, (j > 0 || k > 0) ? 1u : 0u);
            tc_commit_warp(&sh.pvdone[u]);
        }
        tc_commit_warp(&sh.mma_done);          // every MMA above has completed before the teardown
        mbar_wait(&sh.mma_done, 0, kWaitNs);
    } else if (warp >= 4) {
        // =========================================================== loaders
        const int ti = tid - 128;                 // token ti (keys) and channel ti (values)
        const int pp_k = ti >> 6, slot_k = ti & 63;
        auto issue = [&](int k) {
            uint8_t* st = ring + (k % R) * C::STAGE;
            if (k < nt) {                         // key codes of token ti
                const int lp = pg0 + 2 * k + pp_k;
                const int pg = lp < pg1 ? sh.pages[2 * k + pp_k] : -1;
                const bool have = pg >= 0;
                const uint8_t* kb = p.k_codes + (size_t(have ? pg : 0) * p.hkv + h) * (kPage * C::KROW) + slot_k * 16;
#pragma unroll
                for (int c = 0; c < C::KROW / 16; ++c)
                    cp16(st + c * (TILE * 16) + ti * 16, kb + c * (kPage * 16), have);
            } else {                              // value codes of channel ti, both pages
                const int i = k - nt;
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    const int lp = pg0 + 2 * i + pp;
                    const int pg = lp < pg1 ? sh.pages[2 * i + pp] : -1;
                    const bool have = pg >= 0;
                    const uint8_t* vb = p.v_codes + (size_t(have ? pg : 0) * p.hkv + h) * (D * C::VCH);
                    if constexpr (C::VCH >= 16) {
#pragma unroll
                        for (int c = 0; c < C::VCH / 16; ++c)
                            cp16(st + (pp * (C::VCH / 16) + c) * (D * 16) + ti * 16, vb + c * (D * 16) + ti * 16, have);
                    } else {
                        cp8(st + ti * 16 + pp * 8, vb + ti * 8, have);
                    }
                }
            }
        };
        for (int k = 0; k < R - 1; ++k) {
            if (k < 2 * nt) issue(k);
            cp_commit();
        }
        for (int k = 0; k < 2 * nt; ++k) {
            if (k + R - 1 < 2 * nt) issue(k + R - 1);
            cp_commit();
            cp_wait<R - 1>();
            const uint8_t* st = ring + (k % R) * C::STAGE;
            if (k < nt) {
                // ---- key codes of tile i -> int8 operand buffer i&1
                const int i = k;
                uint32_t a[32];
#pragma unroll
                for (int c = 0; c < C::KROW / 16; ++c) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(st + c * (TILE * 16) + ti * 16);
                    unpack_i8<KB>(w4.x, &a[(4 * c + 0) * (8 / KB)]);
                    unpack_i8<KB>(w4.y, &a[(4 * c + 1) * (8 / KB)]);
                    unpack_i8<KB>(w4.z, &a[(4 * c + 2) * (8 / KB)]);
                    unpack_i8<KB>(w4.w, &a[(4 * c + 3) * (8 / KB)]);
                }
                // score MMA of tile i-2 done (waiting on tile i-SB: a later phase of the
                // same barrier cannot complete before this operand is written)
                if (i >= SB) wait(&sh.sfull[(i - SB) % SB], ((i - SB) / SB) & 1);
                if (__any_sync(FULL, !ok)) break;
                tc_fence_after();
                tmem_st32(tbase + lane_off + C::COL_AK + 32 * (i & 1), a);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.kfull[i & 1]);
            } else {
                // ---- value codes of tile j -> bf16 operand buffer j&1
                const int j = k - nt, u = j & 1;
                const int last = nt - 1;
                if (j == 0) wait(&sh.sfull[last % SB], (last / SB) & 1);   // every score MMA done
                if (j == 1) wait(&sh.sfree[last % SB], (last / SB) & 1);   // every score accumulator read
                if (j >= 2) wait(&sh.pvdone[u], ((j - 2) >> 1) & 1);        // ·V MMA of tile j-2 done
                if (__any_sync(FULL, !ok)) break;
                tc_fence_after();
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {      // one page (32 columns) at a time
                    uint32_t a[32];
                    if constexpr (VB == 1) {
                        const uint2 w2 = *reinterpret_cast<const uint2*>(st + ti * 16 + pp * 8);
                        Unpack<1>::word(w2.x, &a[0]);
                        Unpack<1>::word(w2.y, &a[VREG]);
                    } else {
#pragma unroll
                        for (int c = 0; c < VWP / 4; ++c) {
                            const uint4 w4 = *reinterpret_cast<const uint4*>(st + (pp * (VWP / 4) + c) * (D * 16) + ti * 16);
                            Unpack<VB>::word(w4.x, &a[c * 4 * VREG + 0 * VREG]);
                            Unpack<VB>::word(w4.y, &a[c * 4 * VREG + 1 * VREG]);
                            Unpack<VB>::word(w4.z, &a[c * 4 * VREG + 2 * VREG]);
                            Unpack<VB>::word(w4.w, &a[c * 4 * VREG + 3 * VREG]);
                        }
                    }
                    tmem_st32(tbase + lane_off + C::COL_AV + 64 * u + 32 * pp, a);
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.vfull[u]);
            }
        }
        cp_wait_all();
    } else {
        // =========================================================== softmax
        const int t = tid, pp_t = t >> 6, slot_t = t & 63;
        const int kpos_t = pp_t * kPage + kpos_bf16(slot_t, VB);   // position along the ·V K dimension
        auto issue = [&](int k) {                 // metadata of token t: keys in phase 1, values in phase 2
            uint8_t* st = ring + (k % R) * C::STAGE + C::ST_M;
            const int i = k < nt ? k : k - nt;
            const int lp = pg0 + 2 * i + pp_t;
            const int pg = lp < pg1 ? sh.pages[2 * i + pp_t] : -1;
            const bool have = pg >= 0;
            const size_t ph = size_t(have ? pg : 0) * p.hkv + h;
            if (k < nt) cp16(st + t * 16, p.k_meta + (ph * kPage + slot_t) * NKG, have);
            else cp4(st + t * 16, p.v_meta + (ph * kPage + slot_t), have);   // same bytes as the key step
        };
        for (int k = 0; k < R - 1; ++k) {
            if (k < 2 * nt) issue(k);
            cp_commit();
        }
        float qsum[NHC][NKG], qs0[NHC], mloc[NHC];
#pragma unroll
        for (int r = 0; r < NHC; ++r) {
            qs0[r] = sh.qs0[r < g ? r : 0];
            mloc[r] = -INFINITY;
#pragma unroll
            for (int grp = 0; grp < NKG; ++grp) qsum[r][grp] = sh.qsum[r < g ? r : 0][grp];
        }
        // ---- phase 1: scores of every tile, into shared memory
        for (int i = 0; i < nt; ++i) {
            if (i + R - 1 < 2 * nt) issue(i + R - 1);
            cp_commit();
            cp_wait<R - 1>();
            const uint4 km4 = *reinterpret_cast<const uint4*>(ring + (i % R) * C::STAGE + C::ST_M + t * 16);
            const int lp = pg0 + 2 * i + pp_t;
            const bool valid = lp < pg1 && sh.pages[2 * i + pp_t] >= 0 && lp * kPage + slot_t < Lq;
            const uint32_t kmw[NKG] = {km4.x, km4.y, km4.z, km4.w};
            float ksc[NKG], kzp[NKG];
#pragma unroll
            for (int grp = 0; grp < NKG; ++grp) {
                const float2 f = meta_f2(kmw[grp]);
                ksc[grp] = f.x;
                kzp[grp] = KB == 8 ? fmaf(128.0f, f.x, f.y) : f.y;   // folds the -128 code offset
            }
            const int sb = i % SB;
            wait(&sh.sfull[sb], (i / SB) & 1);
            if (__any_sync(FULL, !ok)) break;
            tc_fence_after();
#pragma unroll
            for (int hp = 0; hp < NHC / 2; ++hp) {
                uint32_t ds[24];
#pragma unroll
                for (int c = 0; c < 3; ++c) tmem_ld8(tbase + lane_off + C::COL_S + NS * sb + 24 * hp + 8 * c, &ds[8 * c]);
                tc_wait_ld();
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int r = 2 * hp + rr;
                    float a1 = 0.0f, a2 = 0.0f;
#pragma unroll
                    for (int grp = 0; grp < NKG; ++grp) {
                        const int n0 = 12 * rr + 3 * grp;
                        float dot;
                        if constexpr (KB <= 4) {
                            dot = (float)(int(ds[n0]) * 16384 + int(ds[n0 + 1]) * 128 + int(ds[n0 + 2]));
                        } else {
                            dot = fmaf((float)int(ds[n0]), 16384.0f,
                                       fmaf((float)int(ds[n0 + 1]), 128.0f, (float)int(ds[n0 + 2])));
                        }
                        a1 = fmaf(ksc[grp], dot, a1);
                        a2 = fmaf(kzp[grp], qsum[r][grp], a2);
                    }
                    const float sc = (valid && r < g) ? fmaf(a1, qs0[r], a2) * scale_log2 : -INFINITY;
                    scs[(i * NHC + r) * TILE + t] = sc;
                    mloc[r] = fmaxf(mloc[r], sc);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.sfree[sb]);
        }
        // ---- the split's score maximum per head
        const int bad1 = __any_sync(FULL, !ok);
#pragma unroll
        for (int r = 0; r < NHC; ++r) {
            const float wm = warp_max(mloc[r]);
            if (lane == 0) sh.smax[warp][r] = wm;
        }
        if (lane == 0 && bad1) sh.abort = 1;
        named_sync(1, 128);
        if (sh.abort) ok = false;
        float m[NHC], mu[NHC], l[NHC], pz[NHC];
#pragma unroll
        for (int r = 0; r < NHC; ++r) {
            m[r] = fmaxf(fmaxf(sh.smax[0][r], sh.smax[1][r]), fmaxf(sh.smax[2][r], sh.smax[3][r]));
            mu[r] = (m[r] == -INFINITY) ? 0.0f : m[r];
            l[r] = 0.0f;
            pz[r] = 0.0f;
        }
        // ---- phase 2: P' of every tile
        for (int j = 0; j < nt && ok; ++j) {
            const int k = nt + j, u = j & 1;
            if (k + R - 1 < 2 * nt) issue(k + R - 1);
            cp_commit();
            cp_wait<R - 1>();
            const uint32_t vmw = *reinterpret_cast<const uint32_t*>(ring + (k % R) * C::STAGE + C::ST_M + t * 16);
            const int lp = pg0 + 2 * j + pp_t;
            const bool valid = lp < pg1 && sh.pages[2 * j + pp_t] >= 0 && lp * kPage + slot_t < Lq;
            const float2 vf = meta_f2(vmw);
            const float vsc = valid ? vf.x : 0.0f;
            const float vzp = valid ? vf.y : 0.0f;                   // value codes are exact bf16
            if (j >= 2) wait(&sh.pvdone[u], ((j - 2) >> 1) & 1);     // ·V MMA of tile j-2 read buffer u
            if (__any_sync(FULL, !ok)) break;
            uint8_t* pbu = pb + u * 16 * C::CS_P;
#pragma unroll
            for (int r = 0; r < NHC; ++r) {
                if (r >= g) continue;
                const float pr = ex2(scs[(j * NHC + r) * TILE + t] - mu[r]);
                l[r] += pr;
                pz[r] = fmaf(pr, vzp, pz[r]);
                const float pv = pr * vsc;
                const float hi = __bfloat162float(__float2bfloat16_rn(pv));
                *reinterpret_cast<uint16_t*>(pbu + b_off_bf16(2 * r, kpos_t, C::CS_P)) = bf16_bits(pv);
                *reinterpret_cast<uint16_t*>(pbu + b_off_bf16(2 * r + 1, kpos_t, C::CS_P)) = bf16_bits(pv - hi);
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.pfull[u]);
        }
        cp_wait_all();
        // ---- partial of this split: o for channel t, m, l
        const int last = nt - 1;
        wait(&sh.pvdone[last & 1], (last >> 1) & 1);
        tc_fence_after();
        uint32_t o[16];
        tmem_ld16(tbase + lane_off + C::COL_O, o);
        tc_wait_ld();
#pragma unroll
        for (int r = 0; r < NHC; ++r) {
            const float ls = warp_sum(l[r]);
            const float zs = warp_sum(pz[r]);
            if (lane == 0 && r < g) {
                sh.red[warp][r] = ls;
                sh.red2[warp][r] = zs;
            }
        }
        named_sync(1, 128);
        const bool bad = !ok || sh.abort;
#pragma unroll
        for (int r = 0; r < NHC; ++r) {
            if (r >= g) continue;
            const float z = (sh.red2[0][r] + sh.red2[1][r]) + (sh.red2[2][r] + sh.red2[3][r]);
            const size_t row = row0 + size_t(r) * slots + x;
            ws_o[row * D + t] = bad ? NAN : __uint_as_float(o[2 * r]) + __uint_as_float(o[2 * r + 1]) + z;
            if (t == 0) {
                const float ls = (sh.red[0][r] + sh.red[1][r]) + (sh.red[2][r] + sh.red[3][r]);
                ws_ml[row * 2 + 0] = bad ? 0.0f : m[r];
                ws_ml[row * 2 + 1] = bad ? NAN : ls;
            }
        }
        if (bad && t == 0) atomicAdd(&status[0], 1u);
    }
    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tbase, C::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace kvq

// Persistent decode attention over the quantized cache with register-resident
// tensor-core fragments (sm_100a): head_dim 128, key groups of 32 channels,
// value groups of 128 channels, key/value bit widths in {1, 2, 4, 8}, up to
// 8 query heads per kv-head.
//
// What it computes ("Kuantisasi KV cache mengganggu attention ...", section
// "Error pada key masuk sebelum softmax"): s = q K^T * sm_scale,
// a = softmax(s), o = a V, with dequantization fused into the kernel
// (section "Pertumbuhan cache mengubah trade pada serving").  With
// x^ = c*scale + zero per group:
//   q . k^ = sum_groups ( scale * (q . c)_group + zero * (sum q)_group )
//   o      = sum_t (p_t scale_t) c_t + sum_t p_t zero_t
// Both contractions run on the integer tensor cores over the raw codes:
//  - scores: mma m16n8k32 u8 x s8.  A = key codes (rows = tokens, K = the
//    32 channels of one key group), B = the query of each head split into
//    three int8 limbs a + b/2^7 + c/2^14 times a power of two (2^-20 of the
//    head's largest element), one column per (head, limb).  The limbs are
//    recombined exactly in int32 and the group's fp16 scale applied in fp32.
//  - values: mma m16n8k32 u8 x u8.  A = value codes (rows = channels,
//    K = tokens), B = P' = p * value_scale quantized against the unit's
//    largest P' into three 8-bit limbs (2^-24 of that maximum), one column
//    per (head, limb), recombined in fp32 when the unit is done.
// The newest W positions (bf16 window) run on bf16 mma m16n8k16 with the
// query and the weights as bf16 (high, low) pairs.
//
// Work: the (sequence, kv-head) pairs are cut into units (UP pages of
// quantized tokens, or WU window positions); the units are laid end to end
// and each CTA (one per SM) takes an equal contiguous range, each of its
// consumer warps an equal contiguous share of that.  A producer warp streams
// the units' pages into a ring of shared-memory slots with 1-D bulk copies
// (window rows with 16-byte cp.async into a swizzled layout), completion
// counted on an mbarrier per slot.  Every consumer warp keeps its own online
// softmax state; a pair that spans several warps is merged through shared
// memory, a pair that spans several CTAs through a partial in the workspace
// merged by the CTA that finishes it last (an atomic ticket per pair, reset
// by that CTA).  Every mbarrier wait is bounded.
#pragma once

#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_tc_ptx.cuh"
#include "kvq_mma_ptx.cuh"

namespace kvq {
namespace mma {

using namespace ptx;

constexpr int D = 128;
constexpr int NKG = 4;                         // key groups of 32 channels
constexpr int NW = 8;                          // consumer warps
constexpr int kThreads = 32 * (NW + 1);        // + one producer warp
constexpr int kMaxSlots = 32;
constexpr int kMaxBatch = 4096;                // schedule tables live in shared memory
constexpr int kSmemBudget = 227 * 1024;
constexpr unsigned FULL = 0xffffffffu;
constexpr uint64_t kWaitNs = 1000000000ull;    // bound on every wait: 1 s
constexpr uint64_t kDrainNs = 100000000ull;
constexpr float kLn2 = 0.69314718055994530942f;


// window positions per window unit: about the bytes of a quantized unit
__host__ __device__ constexpr int window_unit(int qbytes) {
    return qbytes >= 64 * 512 ? 64 : (qbytes >= 24 * 512 ? 32 : 16);
}

template <int KB, int VB, int NH>
struct Cfg {
    static constexpr int UP = 2;                         // pages per quantized unit
    static constexpr int TOK = UP * kPage;               // tokens per quantized unit
    static constexpr int HS = NH / 4;                    // heads per thread
    static constexpr int NT = NH == 4 ? 2 : 3;           // 8-column tiles of (head, limb)
    static constexpr int KROW = D * KB / 8;
    static constexpr int KCODES = kPage * KROW;          // one (page, kv-head) block
    static constexpr int KMETA = kPage * NKG * 4;
    static constexpr int VCH = kPage * VB / 8;           // bytes of one channel in one page
    static constexpr int VCODES = D * VCH;
    static constexpr int VMETA = kPage * 4;
    static constexpr int PAGE_BYTES = KCODES + KMETA + VCODES + VMETA;
    static constexpr int OFF_KM = UP * KCODES;
    static constexpr int OFF_VC = OFF_KM + UP * KMETA;
    static constexpr int OFF_VM = OFF_VC + UP * VCODES;
    static constexpr int QBYTES = OFF_VM + UP * VMETA;
    static constexpr int WU = window_unit(QBYTES);
    static constexpr int WROWS = WU * D * 2;             // bytes of the key (or value) rows of a window unit
    static constexpr int SLOT = ((QBYTES > 2 * WROWS ? QBYTES : 2 * WROWS) + 127) & ~127;
    static constexpr int QAREA = NH * 512 + NH * 32;     // per consumer warp: limb / bf16 query staging + scalars
    static_assert(KCODES % 16 == 0 && KMETA % 16 == 0 && VCODES % 16 == 0 && VMETA % 16 == 0, "bulk sizes");
};

struct Head {
    uint64_t full[kMaxSlots];
    uint64_t empty[kMaxSlots];
    int abort;
    int cs, ce, cta_pair0;                 // this CTA's unit range and the pair of its first unit
    int wpair[NW][2];                      // pairs of a warp's incomplete segments, -1 if none
};

__host__ __device__ inline int off_sched() { return (int(sizeof(Head)) + 15) & ~15; }
__host__ __device__ inline int off_qarea(int batch) { return (off_sched() + 8 * (batch + 1) + 127) & ~127; }
// merge partials: per head a row of D outputs, the running maximum and the
// weight sum, padded to PST floats so that every row starts 16-byte aligned
constexpr int PST = D + 4;
template <int NH>
__host__ __device__ constexpr int part_floats() { return NH * PST; }
// a warp's first segment, when another warp began its pair, is parked here
// until the merge: NW partials of g heads
template <int KB, int VB, int NH>
__host__ __device__ inline int off_park(int batch) {
    return (off_qarea(batch) + NW * Cfg<KB, VB, NH>::QAREA + 127) & ~127;
}
template <int KB, int VB, int NH>
__host__ __device__ inline int off_ring(int batch, int g) {
    return (off_park<KB, VB, NH>(batch) + NW * g * PST * 4 + 127) & ~127;
}

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ int rni(float x) {
    int r;
    asm("cvt.rni.s32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
    return v;
}
__device__ __forceinline__ float grp_max(float v) {   // over the 8 lanes that share lane & 3
    v = fmaxf(v, __shfl_xor_sync(FULL, v, 4));
    v = fmaxf(v, __shfl_xor_sync(FULL, v, 8));
    return fmaxf(v, __shfl_xor_sync(FULL, v, 16));
}
__device__ __forceinline__ float grp_sum(float v) {
    v += __shfl_xor_sync(FULL, v, 4);
    v += __shfl_xor_sync(FULL, v, 8);
    return v + __shfl_xor_sync(FULL, v, 16);
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float2 half2f(uint32_t w) {   // {u16 lo, u16 hi} binary16 -> (lo, hi)
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Token (0..31 inside a 32-token step) whose score row `gp` (0..7) holds as
// its i-th value (i = 0..3).  It is the token set that the value fragment of
// lane group gp%4 packs into one register (first half of the step's K for
// gp < 4, second half otherwise), so that the weights of the ·V product are
// found in one lane.
template <int VB>
__device__ __forceinline__ int tmap(int gp, int i) {
    const int t = gp & 3, hi = gp >> 2;
    if constexpr (VB == 1) return t + 4 * hi + 8 * i;
    else if constexpr (VB == 2) return t + 16 * hi + 4 * i;
    else if constexpr (VB == 4) return 8 * t + hi + 2 * i;
    else return 4 * t + 16 * hi + i;
}

// K position (0..31) of channel `ch` (0..31 in its key group) in the score
// MMA: the inverse of the byte layout that the key-fragment unpacking below
// produces (low K half from register a0/a1, high half from a2/a3).
template <int KB>
__host__ __device__ __forceinline__ int kpos(int ch) {
    if constexpr (KB == 4) return 16 * (ch & 1) + 4 * (ch >> 3) + ((ch & 7) >> 1);
    else if constexpr (KB == 8) return ch;
    else if constexpr (KB == 2) return 16 * (ch & 1) + 4 * (2 * (ch >> 4) + ((ch >> 1) & 1)) + ((ch & 15) >> 2);
    else return 16 * ((ch >> 2) & 1) + 4 * (ch & 3) + (ch >> 3);
}

// byte offset of 32-bit word `wi` of key token slot `t` inside a page block
__device__ __forceinline__ uint32_t kword(int t, int wi) { return (wi >> 2) * (kPage * 16) + t * 16 + (wi & 3) * 4; }

// Score A fragment of key group `grp` for rows tA (a0, a2) and tB (a1, a3).
template <int KB>
__device__ __forceinline__ void kfrag(uint32_t kc, int tA, int tB, int grp, int tig, uint32_t (&a)[4]) {
    if constexpr (KB == 4) {
        const uint32_t wA = lds32(kc + kword(tA, 4 * grp + tig)), wB = lds32(kc + kword(tB, 4 * grp + tig));
        a[0] = wA & 0x0F0F0F0Fu;
        a[2] = (wA >> 4) & 0x0F0F0F0Fu;
        a[1] = wB & 0x0F0F0F0Fu;
        a[3] = (wB >> 4) & 0x0F0F0F0Fu;
    } else if constexpr (KB == 8) {
        a[0] = lds32(kc + kword(tA, 8 * grp + tig));
        a[2] = lds32(kc + kword(tA, 8 * grp + 4 + tig));
        a[1] = lds32(kc + kword(tB, 8 * grp + tig));
        a[3] = lds32(kc + kword(tB, 8 * grp + 4 + tig));
    } else if constexpr (KB == 2) {
        const int sh = 4 * (tig & 1);
        const uint32_t wA = lds32(kc + kword(tA, 2 * grp + (tig >> 1)));
        const uint32_t wB = lds32(kc + kword(tB, 2 * grp + (tig >> 1)));
        a[0] = (wA >> sh) & 0x03030303u;
        a[2] = (wA >> (sh + 2)) & 0x03030303u;
        a[1] = (wB >> sh) & 0x03030303u;
        a[3] = (wB >> (sh + 2)) & 0x03030303u;
    } else {
        const uint32_t wA = lds32(kc + kword(tA, grp)), wB = lds32(kc + kword(tB, grp));
        a[0] = (wA >> tig) & 0x01010101u;
        a[2] = (wA >> (tig + 4)) & 0x01010101u;
        a[1] = (wB >> tig) & 0x01010101u;
        a[3] = (wB >> (tig + 4)) & 0x01010101u;
    }
}

// ·V A fragment for channels chA (a0, a2) and chB (a1, a3), 32-token step
// `half` of a page (value codes stored per channel, chunk-major above 16 B).
template <int VB>
__device__ __forceinline__ void vfrag(uint32_t vc, int chA, int chB, int half, int tig, uint32_t (&a)[4]) {
    if constexpr (VB == 2) {
        const uint2 wA = lds64(vc + chA * 16 + 8 * half), wB = lds64(vc + chB * 16 + 8 * half);
        a[0] = (wA.x >> (2 * tig)) & 0x03030303u;
        a[2] = (wA.y >> (2 * tig)) & 0x03030303u;
        a[1] = (wB.x >> (2 * tig)) & 0x03030303u;
        a[3] = (wB.y >> (2 * tig)) & 0x03030303u;
    } else if constexpr (VB == 4) {
        const uint32_t wA = lds32(vc + half * (D * 16) + chA * 16 + 4 * tig);
        const uint32_t wB = lds32(vc + half * (D * 16) + chB * 16 + 4 * tig);
        a[0] = wA & 0x0F0F0F0Fu;
        a[2] = (wA >> 4) & 0x0F0F0F0Fu;
        a[1] = wB & 0x0F0F0F0Fu;
        a[3] = (wB >> 4) & 0x0F0F0F0Fu;
    } else if constexpr (VB == 8) {
        a[0] = lds32(vc + (2 * half) * (D * 16) + chA * 16 + 4 * tig);
        a[2] = lds32(vc + (2 * half + 1) * (D * 16) + chA * 16 + 4 * tig);
        a[1] = lds32(vc + (2 * half) * (D * 16) + chB * 16 + 4 * tig);
        a[3] = lds32(vc + (2 * half + 1) * (D * 16) + chB * 16 + 4 * tig);
    } else {
        const uint32_t wA = lds32(vc + chA * 8 + 4 * half), wB = lds32(vc + chB * 8 + 4 * half);
        a[0] = (wA >> tig) & 0x01010101u;
        a[2] = (wA >> (tig + 4)) & 0x01010101u;
        a[1] = (wB >> tig) & 0x01010101u;
        a[3] = (wB >> (tig + 4)) & 0x01010101u;
    }
}

// q . codes of one key group from its three limb columns (exact in int32 for
// codes below 16; 8-bit codes combine the first two limbs in int32)
template <int KB>
__device__ __forceinline__ float limb_dot(int32_t l0, int32_t l1, int32_t l2) {
    if constexpr (KB <= 4) return (float)(l0 * 16384 + l1 * 128 + l2);
    else return fmaf((float)(l0 * 128 + l1), 128.0f, (float)l2);
}
// P' . codes from the three 8-bit limb columns
template <int VB>
__device__ __forceinline__ float limb_pv(int32_t l0, int32_t l1, int32_t l2) {
    if constexpr (VB <= 4) return fmaf((float)(l0 * 256 + l1), 256.0f, (float)l2);
    else return fmaf(fmaf((float)l0, 256.0f, (float)l1), 256.0f, (float)l2);
}

// swizzle of the 16-byte chunks of window row t: ldmatrix rows (tokens
// 2r or 2r+1 for scores, r or 8+r for ·V) fall in distinct bank groups
__device__ __forceinline__ int wswz(int t) { return (t & 7) ^ ((t >> 3) & 1); }

// ---------------------------------------------------------------- schedule
struct UnitPos {
    int b, h, j, n;
};
// unit u -> sequence b, kv-head h, index j inside the pair, units n of the pair
__device__ __forceinline__ UnitPos locate(const int* S, int B, int H, int u) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (H * S[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    const int n = S[lo + 1] - S[lo], r = u - H * S[lo];
    return {lo, r / n, r % n, n};
}
__device__ __forceinline__ int cta_start(long long c, long long U, long long C) { return (int)((c * U) / C); }
__device__ __forceinline__ int cta_of(long long u, long long U, long long C) { return (int)(((u + 1) * C - 1) / U); }

// ---------------------------------------------------------------- per-thread state
template <int NH>
struct State {
    static constexpr int HS = NH / 4;
    float m[HS], l[HS], pz[HS];
    float o[HS][8][2];     // channels 16*mt + g and 16*mt + g + 8 of head tig (+4)
    bool bad;
    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int hs = 0; hs < HS; ++hs) {
            m[hs] = -INFINITY;
            l[hs] = 0.0f;
            pz[hs] = 0.0f;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) o[hs][mt][0] = o[hs][mt][1] = 0.0f;
        }
        bad = false;
    }
};

// ---------------------------------------------------------------- query preparation
// Query of kv-head h of sequence b: int8 limbs of the (rotated) query in the
// score MMA's K order, staged in the warp's area, then read into the B
// fragments; per head the limb unit (times sm_scale*log2 e) and the sums of
// the rotated query per key group (times the same).
template <int KB, int NH>
__device__ void prep_query(const Params& p, const void* q, int q_bf16, int b, int h, uint8_t* qa, float sl2,
                           int lane, uint32_t (&qb)[NKG][Cfg<KB, 1, NH>::NT][2], float (&cq)[NH / 4],
                           float (&cz)[NH / 4][NKG]) {
    constexpr int NT = Cfg<KB, 1, NH>::NT;
    const int g = p.g;
    int8_t* ql = reinterpret_cast<int8_t*>(qa);                 // [limb][head][group][32]
    float* qs = reinterpret_cast<float*>(qa + NH * 512);         // [head][8]
#pragma unroll 1
    for (int r = 0; r < NH; ++r) {
        float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (r < g) {
            const size_t off = (size_t(b) * p.hq + size_t(h) * g + r) * D + 4 * lane;
            if (q_bf16) {
                const uint2 v = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(q) + off));
                x[0] = bf_lo(v.x);
                x[1] = bf_hi(v.x);
                x[2] = bf_lo(v.y);
                x[3] = bf_hi(v.y);
            } else {
                const float4 v = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(q) + off));
                x[0] = v.x;
                x[1] = v.y;
                x[2] = v.z;
                x[3] = v.w;
            }
            if (p.rotate) rotate_warp<D>(x, p.signs, lane);
        }
        float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
        amax = warp_max(amax);
        float gs = (x[0] + x[1]) + (x[2] + x[3]);
        gs += __shfl_xor_sync(FULL, gs, 1);
        gs += __shfl_xor_sync(FULL, gs, 2);
        gs += __shfl_xor_sync(FULL, gs, 4);                      // lanes 8grp .. 8grp+7: key group grp
        const uint32_t eb = __float_as_uint(amax) >> 23;         // amax < 2^(eb - 126)
        const bool use = eb >= 40;
        const float inv_s0 = use ? __uint_as_float((259u - eb) << 23) : 0.0f;   // 1/s0, s0 = 2^(eb-132)
        if ((lane & 7) == 0) qs[r * 8 + 1 + (lane >> 3)] = gs * sl2;
        if (lane == 0) qs[r * 8] = (use ? __uint_as_float((eb - 19u) << 23) : 0.0f) * sl2;   // s0 * 2^-14
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int ch = 4 * lane + c, grp = ch >> 5;
            const float xs = x[c] * inv_s0;                        // |xs| < 64, exact
            const int a = rni(xs);
            const float r1 = (xs - (float)a) * 128.0f;
            const int bl = rni(r1);
            const float r2 = (r1 - (float)bl) * 128.0f;
            const int cl = rni(r2);
            const int o = grp * 32 + kpos<KB>(ch & 31);
            ql[(0 * NH + r) * 128 + o] = (int8_t)a;
            ql[(1 * NH + r) * 128 + o] = (int8_t)bl;
            ql[(2 * NH + r) * 128 + o] = (int8_t)cl;
        }
    }
    __syncwarp();
    const int n = lane >> 2, tig = lane & 3;
    auto frag = [&](int head, int limb, int grp, int half) -> uint32_t {
        return *reinterpret_cast<const uint32_t*>(ql + (limb * NH + head) * 128 + grp * 32 + half * 16 + 4 * tig);
    };
#pragma unroll
    for (int grp = 0; grp < NKG; ++grp) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            qb[grp][0][hf] = frag(n >> 1, n & 1, grp, hf);
            if constexpr (NH == 4) {
                qb[grp][1][hf] = (n & 1) ? 0u : frag(n >> 1, 2, grp, hf);
            } else {
                qb[grp][1][hf] = frag(4 + (n >> 1), n & 1, grp, hf);
                qb[grp][2][hf] = frag((n >> 1) + 4 * (n & 1), 2, grp, hf);
            }
        }
    }
#pragma unroll
    for (int hs = 0; hs < NH / 4; ++hs) {
        cq[hs] = qs[(tig + 4 * hs) * 8];
#pragma unroll
        for (int grp = 0; grp < NKG; ++grp) cz[hs][grp] = qs[(tig + 4 * hs) * 8 + 1 + grp];
    }
    __syncwarp();
}

// Unrotated query as bf16 (high, low) pairs for the window scores:
// [head][high/low][channel] bf16 in the warp's area.
template <int NH>
__device__ void prep_window_query(const Params& p, const void* q, int q_bf16, int b, int h, uint8_t* qa, int lane) {
    __nv_bfloat16* wq = reinterpret_cast<__nv_bfloat16*>(qa);
    const int g = p.g;
    __syncwarp();
#pragma unroll 1
    for (int r = 0; r < NH; ++r) {
        float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (r < g) {
            const size_t off = (size_t(b) * p.hq + size_t(h) * g + r) * D + 4 * lane;
            if (q_bf16) {
                const uint2 v = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(q) + off));
                x[0] = bf_lo(v.x);
                x[1] = bf_hi(v.x);
                x[2] = bf_lo(v.y);
                x[3] = bf_hi(v.y);
            } else {
                const float4 v = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(q) + off));
                x[0] = v.x;
                x[1] = v.y;
                x[2] = v.z;
                x[3] = v.w;
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(x[c]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(x[c] - __bfloat162float(hi));
            wq[(r * 2 + 0) * D + 4 * lane + c] = hi;
            wq[(r * 2 + 1) * D + 4 * lane + c] = lo;
        }
    }
    __syncwarp();
}

// ---------------------------------------------------------------- the kernel
template <int KB, int VB, int NH>
__global__ void __launch_bounds__(kThreads, 1)
decode_mma_kernel(const Params p, const void* __restrict__ q, const int q_bf16, const int32_t* __restrict__ lens,
                  const int max_len, const float sl2, float* __restrict__ out, float* __restrict__ lse,
                  float* __restrict__ part, uint32_t* __restrict__ tickets, const int R,
                  unsigned int* __restrict__ status) {
    using C = Cfg<KB, VB, NH>;
    constexpr int HS = C::HS, NT = C::NT, TOK = C::TOK, WU = C::WU;
    extern __shared__ __align__(1024) uint8_t smem[];
    Head& hd = *reinterpret_cast<Head*>(smem);
    const int B = p.batch, H = p.hkv, g = p.g;
    int* S = reinterpret_cast<int*>(smem + off_sched());    // [B+1] units of one pair of sequences < b
    int* LB = S + (B + 1);                                    // [B] clamped lengths  (S, LB: 8(B+1) bytes)
    uint8_t* qarea = smem + off_qarea(B);
    float* park = reinterpret_cast<float*>(smem + off_park<KB, VB, NH>(B));   // [NW][g][PST]
    uint8_t* ring = smem + off_ring<KB, VB, NH>(B, p.g);
    const uint32_t ring_s = smem_u32(ring);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = p.W;

    // ---- schedule: units per pair of each sequence, prefix over sequences
    for (int b = tid; b < B; b += kThreads) {
        const int L = max(0, min(lens[b], max_len));
        LB[b] = L;
        const int wl = min(W, L), lq = L - wl;
        S[b + 1] = L == 0 ? 1 : (lq + TOK - 1) / TOK + (wl + WU - 1) / WU;
    }
    if (tid == 0) {
        for (int i = 0; i < R; ++i) {
            mbar_init(&hd.full[i], 1);
            mbar_init(&hd.empty[i], 1);
        }
        mbar_fence_init();
        hd.abort = 0;
    }
    __syncthreads();
    if (warp == 0) {
        int run = 0;
        for (int base = 0; base < B; base += 32) {
            int v = base + lane < B ? S[base + lane + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(FULL, v, o);
                if (lane >= o) v += t;
            }
            if (base + lane < B) S[base + lane + 1] = run + v;
            run += __shfl_sync(FULL, v, 31);
        }
        if (lane == 0) S[0] = 0;
    }
    __syncthreads();
    // every active CTA gets at least one unit (U >= 1: a sequence has at least one unit per kv-head)
    const long long U = (long long)H * S[B], NC = min((long long)gridDim.x, U);
    const int cta = blockIdx.x;
    const int cs = cta < NC ? cta_start(cta, U, NC) : 0, ce = cta < NC ? cta_start(cta + 1, U, NC) : 0;
    const int len = ce - cs, base_n = len / NW, rem = len % NW;
    if (tid == 0) {
        hd.cs = cs;
        hd.ce = ce;
        if (len > 0) {
            const UnitPos u0 = locate(S, B, H, cs);
            hd.cta_pair0 = u0.b * H + u0.h;
        } else {
            hd.cta_pair0 = -1;
        }
    }
    if (tid < NW * 2) hd.wpair[tid >> 1][tid & 1] = -1;
    __syncthreads();
    if (len <= 0) return;

    auto wstart = [&](int w) { return cs + w * base_n + min(w, rem); };
    auto wsize = [&](int w) { return base_n + (w < rem ? 1 : 0); };
    auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&hd.abort) != 0; };
    // warp-collective bounded wait: every lane gets the same answer
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
        bool ok = !aborted() && mbar_wait(bar, parity, kWaitNs);
        ok = __all_sync(FULL, ok);
        if (!ok && lane == 0 && atomicExch(&hd.abort, 1) == 0) atomicAdd(&status[0], 1u);
        return ok;
    };

    if (warp == NW) {
        // ============================================================ producer
        int issued = 0;
        for (int s0 = 0; s0 < len; s0 += 32) {
            if (__any_sync(FULL, aborted())) break;
            // lane i prepares step s0 + i: which unit, which pages, how many bytes
            int kind = 0, ub = 0, uh = 0, pg0 = -1, pg1 = -1, w0 = 0, cnt = 0;
            uint32_t bytes = 0;
            const int s = s0 + lane;
            if (s < len) {
                const int w = s % NW, k = s / NW;
                const UnitPos u = locate(S, B, H, wstart(w) + k);
                ub = u.b;
                uh = u.h;
                const int L = LB[u.b], wl = min(W, L), lq = L - wl, nq = (lq + TOK - 1) / TOK;
                if (L == 0) {
                    kind = 0;
                } else if (u.j < nq) {
                    kind = 1;
                    const int lp = u.j * C::UP;
                    pg0 = lp * kPage < lq ? phys_page(p, u.b, lp) : -1;
                    pg1 = (lp + 1) * kPage < lq ? phys_page(p, u.b, lp + 1) : -1;
                    bytes = (pg0 >= 0 ? C::PAGE_BYTES : 0) + (pg1 >= 0 ? C::PAGE_BYTES : 0);
                } else {
                    kind = 2;
                    w0 = lq + (u.j - nq) * WU;
                    cnt = min(WU, L - w0);
                }
            }
            const int n_here = min(32, len - s0);
            for (int i = 0; i < n_here; ++i) {
                const int st = s0 + i;
                const int k_ = __shfl_sync(FULL, kind, i);
                const int b_ = __shfl_sync(FULL, ub, i), h_ = __shfl_sync(FULL, uh, i);
                const int p0 = __shfl_sync(FULL, pg0, i), p1 = __shfl_sync(FULL, pg1, i);
                const int w0_ = __shfl_sync(FULL, w0, i), cnt_ = __shfl_sync(FULL, cnt, i);
                const uint32_t by = __shfl_sync(FULL, bytes, i);
                const int slot = st % R;
                if (st >= R && !wait_bar(&hd.empty[slot], ((st / R) - 1) & 1)) break;
                uint8_t* sl = ring + size_t(slot) * C::SLOT;
                if (k_ == 1) {
                    if (lane == 0) mbar_arrive_expect_tx(&hd.full[slot], by);
                    __syncwarp();
                    if (lane < 4 * C::UP) {
                        const int e = lane >> 2, part_ = lane & 3;
                        const int pg = e ? p1 : p0;
                        if (pg >= 0) {
                            const size_t blk = size_t(pg) * H + h_;
                            const void* src;
                            uint8_t* dst;
                            uint32_t nb;
                            if (part_ == 0) {
                                src = p.k_codes + blk * C::KCODES;
                                dst = sl + e * C::KCODES;
                                nb = C::KCODES;
                            } else if (part_ == 1) {
                                src = p.k_meta + blk * (kPage * NKG);
                                dst = sl + C::OFF_KM + e * C::KMETA;
                                nb = C::KMETA;
                            } else if (part_ == 2) {
                                src = p.v_codes + blk * C::VCODES;
                                dst = sl + C::OFF_VC + e * C::VCODES;
                                nb = C::VCODES;
                            } else {
                                src = p.v_meta + blk * kPage;
                                dst = sl + C::OFF_VM + e * C::VMETA;
                                nb = C::VMETA;
                            }
                            bulk_g2s(dst, src, nb, &hd.full[slot]);
                        }
                    }
                } else if (k_ == 2) {
                    // WU rows of keys then values, 16 chunks of 16 bytes each; rows past
                    // the window's end are zero-filled (their weights are 0, and the ·V
                    // product must not meet non-finite values)
                    const size_t rb = (size_t(b_) * H + h_) * size_t(W);
                    const uint32_t base = ring_s + uint32_t(slot) * C::SLOT;
                    for (int idx = lane; idx < 2 * WU * 16; idx += 32) {
                        const int kv = idx / (WU * 16), rem_ = idx % (WU * 16);
                        const int row = rem_ >> 4, c = rem_ & 15;
                        const bool have = row < cnt_;
                        const __nv_bfloat16* src = (kv ? p.v_win : p.k_win) +
                                                   (rb + size_t(have ? (w0_ + row) % W : 0)) * D + c * 8;
                        cp16_zfill(base + kv * C::WROWS + row * (D * 2) + ((c ^ wswz(row)) << 4), src, have);
                    }
                    cp_async_arrive(&hd.full[slot]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive_plain(&hd.full[slot]);
                } else {
                    if (lane == 0) mbar_arrive_plain(&hd.full[slot]);
                }
                issued = st + 1;
            }
        }
        cp_async_wait_all();
        if (aborted()) {
            // nothing may still be copying into shared memory when the CTA exits
            for (int st = max(0, issued - R); st < issued; ++st)
                mbar_wait(&hd.full[st % R], (st / R) & 1, kDrainNs);
        }
    } else {
        // ============================================================ consumers
        const int w = warp, g8 = lane >> 2, tig = lane & 3;
        const int nunits = wsize(w);
        uint8_t* qa = qarea + w * C::QAREA;
        State<NH> st;
        st.reset();
        int first_pair = -1, last_pair = -1;

        // normalized output and lse of heads tig (+4) of kv-head h of sequence b
        auto write_final = [&](const State<NH>& x, int b, int h) {
#pragma unroll
            for (int hs = 0; hs < HS; ++hs) {
                const float lt = grp_sum(x.l[hs]), zt = grp_sum(x.pz[hs]);
                const int r = tig + 4 * hs;
                if (r >= g) continue;
                const size_t row = size_t(b) * p.hq + size_t(h) * g + r;
                const float inv = lt > 0.0f ? 1.0f / lt : 0.0f;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    out[row * D + 16 * mt + g8] = x.bad ? NAN : (x.o[hs][mt][0] + zt) * inv;
                    out[row * D + 16 * mt + g8 + 8] = x.bad ? NAN : (x.o[hs][mt][1] + zt) * inv;
                }
                if (lse && g8 == 0)
                    lse[row] = x.bad ? NAN : (lt > 0.0f ? (x.m[hs] + log2f(lt)) * kLn2 : -INFINITY);
            }
        };
        // unnormalized partial: per head D outputs (including the zero-point
        // term), the running maximum (log2 domain) and the weight sum
        auto store_partial = [&](const State<NH>& x, float* dst) {
#pragma unroll
            for (int hs = 0; hs < HS; ++hs) {
                const float lt = grp_sum(x.l[hs]), zt = grp_sum(x.pz[hs]);
                const int r = tig + 4 * hs;
                if (r >= g) continue;
                float* d = dst + r * PST;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    d[16 * mt + g8] = x.bad ? NAN : x.o[hs][mt][0] + zt;
                    d[16 * mt + g8 + 8] = x.bad ? NAN : x.o[hs][mt][1] + zt;
                }
                if (g8 == 0) {
                    d[D] = x.bad ? 0.0f : x.m[hs];
                    d[D + 1] = x.bad ? NAN : lt;
                }
            }
        };
        // Merge the partials of pair P held by warps w.. of this CTA; output it
        // if the pair lies inside the CTA, else hand a partial to the CTA that
        // finishes the pair last.  Lane l owns channels 4l .. 4l+3.
        auto merge_pair = [&](int P, int w0) {
            const float* src[NW];
            int np = 0;
            for (int ww = w0; ww < NW; ++ww) {
                const int slp = hd.wpair[ww][0] == P ? 0 : (hd.wpair[ww][1] == P ? 1 : -1);
                if (slp < 0) break;
                src[np++] = (slp == 0 ? park : reinterpret_cast<const float*>(ring)) + ww * g * PST;
            }
            const int b = P / H, h = P % H;
            const int n = S[b + 1] - S[b];
            const long long u0 = (long long)H * S[b] + (long long)h * n;
            const bool inside = u0 >= cs && u0 + n <= ce;
            float* gdst = part + (size_t(cta) * 2 + (P == hd.cta_pair0 ? 0 : 1)) * part_floats<NH>();
            for (int r = 0; r < g; ++r) {
                float M = -INFINITY;
                for (int i = 0; i < np; ++i) M = fmaxf(M, src[i][r * PST + D]);
                const float mu = M == -INFINITY ? 0.0f : M;
                float Ls = 0.0f, O[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                for (int i = 0; i < np; ++i) {
                    const float* pr = src[i] + r * PST;
                    const float wgt = pr[D] == -INFINITY ? 0.0f : ex2(pr[D] - mu);
                    Ls = fmaf(pr[D + 1], wgt, Ls);
                    const float4 v = *reinterpret_cast<const float4*>(pr + 4 * lane);
                    O[0] = fmaf(v.x, wgt, O[0]);
                    O[1] = fmaf(v.y, wgt, O[1]);
                    O[2] = fmaf(v.z, wgt, O[2]);
                    O[3] = fmaf(v.w, wgt, O[3]);
                }
                if (inside) {
                    const size_t row = size_t(b) * p.hq + size_t(h) * g + r;
                    const float inv = Ls > 0.0f ? 1.0f / Ls : 0.0f;
                    *reinterpret_cast<float4*>(out + row * D + 4 * lane) =
                        make_float4(O[0] * inv, O[1] * inv, O[2] * inv, O[3] * inv);
                    if (lse && lane == 0) lse[row] = Ls > 0.0f ? (M + log2f(Ls)) * kLn2 : (Ls == 0.0f ? -INFINITY : NAN);
                } else {
                    *reinterpret_cast<float4*>(gdst + r * PST + 4 * lane) = make_float4(O[0], O[1], O[2], O[3]);
                    if (lane == 0) {
                        gdst[r * PST + D] = M;
                        gdst[r * PST + D + 1] = Ls;
                    }
                }
            }
            if (inside) return;
            // ---- hand over: the CTA that arrives last merges every CTA's partial of P
            __threadfence();
            __syncwarp();
            unsigned t = 0;
            if (lane == 0) t = atomicAdd(&tickets[P], 1u);
            t = __shfl_sync(FULL, t, 0);
            const int ca = cta_of(u0, U, NC), cb = cta_of(u0 + n - 1, U, NC);
            const unsigned need = unsigned(cb - ca);
            if (t > need) {
                if (lane == 0) atomicAdd(&status[1], 1u);
                return;
            }
            if (t != need) return;
            __threadfence();
            for (int r = 0; r < g; ++r) {
                float M = -INFINITY;
                for (int c = ca; c <= cb; ++c) {
                    const UnitPos f = locate(S, B, H, cta_start(c, U, NC));
                    const float* pr = part + (size_t(c) * 2 + (f.b * H + f.h == P ? 0 : 1)) * part_floats<NH>() +
                                      r * PST;
                    M = fmaxf(M, __ldcg(pr + D));
                }
                const float mu = M == -INFINITY ? 0.0f : M;
                float Ls = 0.0f, O[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                for (int c = ca; c <= cb; ++c) {
                    const UnitPos f = locate(S, B, H, cta_start(c, U, NC));
                    const float* pr = part + (size_t(c) * 2 + (f.b * H + f.h == P ? 0 : 1)) * part_floats<NH>() +
                                      r * PST;
                    const float mc = __ldcg(pr + D);
                    const float wgt = mc == -INFINITY ? 0.0f : ex2(mc - mu);
                    Ls = fmaf(__ldcg(pr + D + 1), wgt, Ls);
                    const float4 v = __ldcg(reinterpret_cast<const float4*>(pr + 4 * lane));
                    O[0] = fmaf(v.x, wgt, O[0]);
                    O[1] = fmaf(v.y, wgt, O[1]);
                    O[2] = fmaf(v.z, wgt, O[2]);
                    O[3] = fmaf(v.w, wgt, O[3]);
                }
                const size_t row = size_t(b) * p.hq + size_t(h) * g + r;
                const float inv = Ls > 0.0f ? 1.0f / Ls : 0.0f;
                *reinterpret_cast<float4*>(out + row * D + 4 * lane) =
                    make_float4(O[0] * inv, O[1] * inv, O[2] * inv, O[3] * inv);
                if (lse && lane == 0) lse[row] = Ls > 0.0f ? (M + log2f(Ls)) * kLn2 : (Ls == 0.0f ? -INFINITY : NAN);
            }
            if (lane == 0) tickets[P] = 0u;       // ready for the next call
        };

        if (nunits > 0) {
            UnitPos pos = locate(S, B, H, wstart(w));
            int seg_j0 = pos.j;
            uint32_t qb[NKG][NT][2];
            float cq[HS], cz[HS][NKG];
            bool wq_ready = false;
            prep_query<KB, NH>(p, q, q_bf16, pos.b, pos.h, qa, sl2, lane, qb, cq, cz);
            for (int k = 0; k < nunits; ++k) {
                const int s = k * NW + w, slot = s % R;
                const int L = LB[pos.b], wl = min(W, L), lq = L - wl, nq = (lq + TOK - 1) / TOK;
                const uint32_t sl = ring_s + uint32_t(slot) * C::SLOT;
                const bool kind_q = L > 0 && pos.j < nq;
                const bool kind_w = L > 0 && pos.j >= nq;
                int pres0 = 0, pres1 = 0;
                if (kind_q) {
                    const int lp = pos.j * C::UP;
                    pres0 = lp * kPage < lq && phys_page(p, pos.b, lp) >= 0;
                    pres1 = (lp + 1) * kPage < lq && phys_page(p, pos.b, lp + 1) >= 0;
                }
                if (kind_w && !wq_ready) {
                    prep_window_query<NH>(p, q, q_bf16, pos.b, pos.h, qa, lane);
                    wq_ready = true;
                }
                const bool ok = wait_bar(&hd.full[slot], (s / R) & 1);
                if (!ok) st.bad = true;
                if (ok && kind_q) {
                    // ---------------------------------------------- quantized unit
                    const int tok0 = pos.j * TOK;
                    float sc[HS][2 * C::UP][4];
#pragma unroll
                    for (int s4 = 0; s4 < 2 * C::UP; ++s4) {
                        const int e = s4 >> 1, o32 = (s4 & 1) * 32;
                        const uint32_t kc = sl + e * C::KCODES, km = sl + C::OFF_KM + e * C::KMETA;
                        const bool pres = e ? pres1 : pres0;
#pragma unroll
                        for (int j2 = 0; j2 < 2; ++j2) {
                            const int tA = o32 + tmap<VB>(g8, 2 * j2), tB = o32 + tmap<VB>(g8, 2 * j2 + 1);
                            const uint4 mA = lds128(km + tA * 16), mB = lds128(km + tB * 16);
                            const uint32_t mAw[4] = {mA.x, mA.y, mA.z, mA.w}, mBw[4] = {mB.x, mB.y, mB.z, mB.w};
                            float accA[HS], accB[HS], zA[HS], zB[HS];
#pragma unroll
                            for (int hs = 0; hs < HS; ++hs) accA[hs] = accB[hs] = zA[hs] = zB[hs] = 0.0f;
#pragma unroll
                            for (int grp = 0; grp < NKG; ++grp) {
                                uint32_t a[4];
                                kfrag<KB>(kc, tA, tB, grp, tig, a);
                                int32_t d[NT][4];
#pragma unroll
                                for (int nt = 0; nt < NT; ++nt) {
                                    d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0;
                                    mma_u8s8(d[nt], a, qb[grp][nt][0], qb[grp][nt][1]);
                                }
                                const float2 fA = half2f(mAw[grp]), fB = half2f(mBw[grp]);
#pragma unroll
                                for (int hs = 0; hs < HS; ++hs) {
                                    const int n0 = NH == 4 ? 0 : hs;              // (l0, l1) tile of this head
                                    const int c2 = NH == 4 ? 0 : hs;              // column of l2 in the last tile
                                    const float dA = limb_dot<KB>(d[n0][0], d[n0][1], d[NT - 1][c2]);
                                    const float dB = limb_dot<KB>(d[n0][2], d[n0][3], d[NT - 1][2 + c2]);
                                    accA[hs] = fmaf(fA.x, dA, accA[hs]);
                                    accB[hs] = fmaf(fB.x, dB, accB[hs]);
                                    zA[hs] = fmaf(fA.y, cz[hs][grp], zA[hs]);
                                    zB[hs] = fmaf(fB.y, cz[hs][grp], zB[hs]);
                                }
                            }
                            const bool vA = pres && tok0 + e * kPage + tA < lq;
                            const bool vB = pres && tok0 + e * kPage + tB < lq;
#pragma unroll
                            for (int hs = 0; hs < HS; ++hs) {
                                sc[hs][s4][2 * j2] = vA ? fmaf(accA[hs], cq[hs], zA[hs]) : -INFINITY;
                                sc[hs][s4][2 * j2 + 1] = vB ? fmaf(accB[hs], cq[hs], zB[hs]) : -INFINITY;
                            }
                        }
                    }
                    // ---- online softmax over the unit; P' limbs
                    float alpha[HS], pscale[HS];
                    uint32_t pl[HS][2 * C::UP][3];
#pragma unroll
                    for (int hs = 0; hs < HS; ++hs) {
                        float mx = -INFINITY;
#pragma unroll
                        for (int s4 = 0; s4 < 2 * C::UP; ++s4)
#pragma unroll
                            for (int i = 0; i < 4; ++i) mx = fmaxf(mx, sc[hs][s4][i]);
                        mx = grp_max(mx);
                        const float mn = fmaxf(st.m[hs], mx);
                        alpha[hs] = mn == -INFINITY ? 1.0f : ex2(st.m[hs] - mn);
                        st.m[hs] = mn;
                        const float mu = mn == -INFINITY ? 0.0f : mn;
                        float ls = 0.0f, zs = 0.0f, pm = 0.0f;
                        float pp[2 * C::UP][4];
#pragma unroll
                        for (int s4 = 0; s4 < 2 * C::UP; ++s4) {
                            const int e = s4 >> 1, o32 = (s4 & 1) * 32;
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                // value metadata of the token; masked tokens (score -inf) get weight 0
                                // and none of their (possibly stale) metadata
                                const int t = o32 + tmap<VB>(g8, i);
                                const float2 f = half2f(lds32(sl + C::OFF_VM + e * C::VMETA + t * 4));
                                const bool v = sc[hs][s4][i] != -INFINITY;
                                const float pr = v ? ex2(sc[hs][s4][i] - mu) : 0.0f;
                                ls += pr;
                                zs = v ? fmaf(pr, f.y, zs) : zs;
                                pp[s4][i] = v ? pr * f.x : 0.0f;
                                pm = fmaxf(pm, pp[s4][i]);
                            }
                        }
                        st.l[hs] = fmaf(st.l[hs], alpha[hs], ls);
                        st.pz[hs] = fmaf(st.pz[hs], alpha[hs], zs);
                        pm = grp_max(pm);
                        const float inv = pm > 0.0f ? 16777215.0f / pm : 0.0f;
                        pscale[hs] = pm * (1.0f / 16777215.0f);
#pragma unroll
                        for (int s4 = 0; s4 < 2 * C::UP; ++s4) {
                            uint32_t x[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) x[i] = min(__float2uint_rn(pp[s4][i] * inv), 16777215u);
                            const uint32_t u01 = __byte_perm(x[0], x[1], 0x5140), u23 = __byte_perm(x[2], x[3], 0x5140);
                            const uint32_t v01 = __byte_perm(x[0], x[1], 0x0062), v23 = __byte_perm(x[2], x[3], 0x0062);
                            pl[hs][s4][0] = __byte_perm(v01, v23, 0x5410);   // limb 0: bits 16..23
                            pl[hs][s4][1] = __byte_perm(u01, u23, 0x7632);   // limb 1: bits 8..15
                            pl[hs][s4][2] = __byte_perm(u01, u23, 0x5410);   // limb 2: bits 0..7
                        }
                    }
                    // ---- ·V: B fragments of P' from the lanes that own the tokens
                    uint32_t bq[2 * C::UP][NT][2];
                    const int srcA = 4 * tig + (g8 >> 1), odd = g8 & 1;
#pragma unroll
                    for (int s4 = 0; s4 < 2 * C::UP; ++s4) {
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int src = srcA + 16 * hf;
                            const uint32_t a0 = __shfl_sync(FULL, pl[0][s4][0], src);
                            const uint32_t a1 = __shfl_sync(FULL, pl[0][s4][1], src);
                            const uint32_t a2 = __shfl_sync(FULL, pl[0][s4][2], src);
                            bq[s4][0][hf] = odd ? a1 : a0;
                            if constexpr (NH == 4) {
                                bq[s4][1][hf] = odd ? 0u : a2;
                            } else {
                                const uint32_t c0 = __shfl_sync(FULL, pl[HS - 1][s4][0], src);
                                const uint32_t c1 = __shfl_sync(FULL, pl[HS - 1][s4][1], src);
                                const uint32_t c2 = __shfl_sync(FULL, pl[HS - 1][s4][2], src);
                                bq[s4][1][hf] = odd ? c1 : c0;
                                bq[s4][2][hf] = odd ? c2 : a2;
                            }
                        }
                    }
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        const int chA = 16 * mt + g8, chB = chA + 8;
                        int32_t acc[NT][4];
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;
#pragma unroll
                        for (int s4 = 0; s4 < 2 * C::UP; ++s4) {
                            uint32_t a[4];
                            vfrag<VB>(sl + C::OFF_VC + (s4 >> 1) * C::VCODES, chA, chB, s4 & 1, tig, a);
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) mma_u8u8(acc[nt], a, bq[s4][nt][0], bq[s4][nt][1]);
                        }
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs) {
                            const int n0 = NH == 4 ? 0 : hs, c2 = NH == 4 ? 0 : hs;
                            const float xA = limb_pv<VB>(acc[n0][0], acc[n0][1], acc[NT - 1][c2]);
                            const float xB = limb_pv<VB>(acc[n0][2], acc[n0][3], acc[NT - 1][2 + c2]);
                            st.o[hs][mt][0] = fmaf(xA, pscale[hs], st.o[hs][mt][0] * alpha[hs]);
                            st.o[hs][mt][1] = fmaf(xB, pscale[hs], st.o[hs][mt][1] * alpha[hs]);
                        }
                    }
                } else if (ok && kind_w) {
                    // ---------------------------------------------- window unit
                    constexpr int NB = WU / 16;
                    const int w0 = lq + (pos.j - nq) * WU, cnt = min(WU, L - w0);
                    const __nv_bfloat16* wq = reinterpret_cast<const __nv_bfloat16*>(qa);
                    const uint32_t kbase = sl, vbase = sl + C::WROWS;
                    float sw[HS][NB][2];
#pragma unroll
                    for (int bb = 0; bb < NB; ++bb) {
                        float d[HS][4];
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs) d[hs][0] = d[hs][1] = d[hs][2] = d[hs][3] = 0.0f;
                        const int mi = lane >> 3, r = lane & 7;
                        const int tq = 16 * bb + 2 * r + (mi & 1);
#pragma unroll
                        for (int s8 = 0; s8 < 8; ++s8) {
                            uint32_t a[4];
                            const int ch = 2 * s8 + (mi >> 1);
                            ldsm_x4(a, kbase + tq * (D * 2) + ((ch ^ wswz(tq)) << 4));
#pragma unroll
                            for (int hs = 0; hs < HS; ++hs) {
                                const int head = (g8 >> 1) + 4 * hs, hl = g8 & 1;
                                const __nv_bfloat16* qq = wq + (head * 2 + hl) * D + 16 * s8 + 2 * tig;
                                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(qq);
                                const uint32_t b1 = *reinterpret_cast<const uint32_t*>(qq + 8);
                                mma_bf16(d[hs], a, b0, b1);
                            }
                        }
                        const int t0 = 16 * bb + 2 * g8;
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs) {
                            sw[hs][bb][0] = t0 < cnt ? (d[hs][0] + d[hs][1]) * sl2 : -INFINITY;
                            sw[hs][bb][1] = t0 + 1 < cnt ? (d[hs][2] + d[hs][3]) * sl2 : -INFINITY;
                        }
                    }
                    float alpha[HS];
                    uint32_t phi[HS][NB], plo[HS][NB];
#pragma unroll
                    for (int hs = 0; hs < HS; ++hs) {
                        float mx = -INFINITY;
#pragma unroll
                        for (int bb = 0; bb < NB; ++bb) mx = fmaxf(mx, fmaxf(sw[hs][bb][0], sw[hs][bb][1]));
                        mx = grp_max(mx);
                        const float mn = fmaxf(st.m[hs], mx);
                        alpha[hs] = mn == -INFINITY ? 1.0f : ex2(st.m[hs] - mn);
                        st.m[hs] = mn;
                        const float mu = mn == -INFINITY ? 0.0f : mn;
                        float ls = 0.0f;
#pragma unroll
                        for (int bb = 0; bb < NB; ++bb) {
                            const float p0 = sw[hs][bb][0] == -INFINITY ? 0.0f : ex2(sw[hs][bb][0] - mu);
                            const float p1 = sw[hs][bb][1] == -INFINITY ? 0.0f : ex2(sw[hs][bb][1] - mu);
                            ls += p0 + p1;
                            phi[hs][bb] = pack_bf16(p0, p1);
                            plo[hs][bb] = pack_bf16(p0 - bf_lo(phi[hs][bb]), p1 - bf_hi(phi[hs][bb]));
                        }
                        st.l[hs] = fmaf(st.l[hs], alpha[hs], ls);
                        st.pz[hs] *= alpha[hs];
                    }
                    uint32_t bv[NB][HS][2];
                    const int srcA = 4 * tig + (g8 >> 1), odd = g8 & 1;
#pragma unroll
                    for (int bb = 0; bb < NB; ++bb)
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs)
#pragma unroll
                            for (int hf = 0; hf < 2; ++hf) {
                                const uint32_t x0 = __shfl_sync(FULL, phi[hs][bb], srcA + 16 * hf);
                                const uint32_t x1 = __shfl_sync(FULL, plo[hs][bb], srcA + 16 * hf);
                                bv[bb][hs][hf] = odd ? x1 : x0;
                            }
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        float dv[HS][4];
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs) dv[hs][0] = dv[hs][1] = dv[hs][2] = dv[hs][3] = 0.0f;
                        const int mi = lane >> 3, r = lane & 7;
#pragma unroll
                        for (int bb = 0; bb < NB; ++bb) {
                            uint32_t a[4];
                            const int tv = 16 * bb + r + 8 * (mi >> 1), ch = 2 * mt + (mi & 1);
                            ldsm_x4_t(a, vbase + tv * (D * 2) + ((ch ^ wswz(tv)) << 4));
#pragma unroll
                            for (int hs = 0; hs < HS; ++hs) mma_bf16(dv[hs], a, bv[bb][hs][0], bv[bb][hs][1]);
                        }
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs) {
                            st.o[hs][mt][0] = fmaf(st.o[hs][mt][0], alpha[hs], dv[hs][0] + dv[hs][1]);
                            st.o[hs][mt][1] = fmaf(st.o[hs][mt][1], alpha[hs], dv[hs][2] + dv[hs][3]);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_plain(&hd.empty[slot]);

                // ---- end of a segment: the pair is done, or the warp's range ends
                const bool pair_end = pos.j + 1 == pos.n, last_unit = k + 1 == nunits;
                if (pair_end || last_unit) {
                    const int pair = pos.b * H + pos.h;
                    if (seg_j0 == 0 && pair_end) {            // the whole pair: final output
                        write_final(st, pos.b, pos.h);
                        st.reset();
                    } else if (!last_unit) {                  // the warp's first segment, begun by another warp
                        store_partial(st, park + w * g * PST);
                        first_pair = pair;
                        st.reset();
                    } else {                                  // the warp's last segment, taken up by another
                        last_pair = pair;
                    }
                }
                // ---- next unit
                if (!pair_end) {
                    ++pos.j;
                } else if (!last_unit) {
                    pos.j = 0;
                    if (++pos.h == H) {
                        pos.h = 0;
                        ++pos.b;
                    }
                    pos.n = S[pos.b + 1] - S[pos.b];
                    seg_j0 = 0;
                    wq_ready = false;
                    prep_query<KB, NH>(p, q, q_bf16, pos.b, pos.h, qa, sl2, lane, qb, cq, cz);
                }
            }
        }

        // ---- merge of pairs split between warps (and CTAs); the ring is free now
        named_barrier(1, NW * 32);
        float* pbase = reinterpret_cast<float*>(ring);
        if (last_pair >= 0) store_partial(st, pbase + w * g * PST);
        if (lane == 0) {            // slot 0: the parked first segment, slot 1: the final segment
            hd.wpair[w][0] = first_pair;
            hd.wpair[w][1] = last_pair;
        }
        named_barrier(1, NW * 32);
#pragma unroll 1
        for (int sl = 0; sl < 2; ++sl) {
            const int P = hd.wpair[w][sl];
            if (P < 0) continue;
            if (w > 0 && (hd.wpair[w - 1][0] == P || hd.wpair[w - 1][1] == P)) continue;   // not the owner
            merge_pair(P, w);
        }
    }
}

}  // namespace mma
}  // namespace kvq

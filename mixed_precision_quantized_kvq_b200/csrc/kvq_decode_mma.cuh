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
// Work: the (sequence, kv-head) pairs are cut into units (one page of
// quantized tokens, or WU window positions); the units are laid end to end,
// each CTA (one per SM) takes an equal contiguous range and each of its warps
// an equal contiguous share of that.  Every warp streams its own units
// through a private ring of shared-memory slots, issuing the copies (1-D bulk
// copies for pages, 16-byte cp.async into a swizzled layout for window rows)
// two units ahead of the one it computes, with completion counted on an
// mbarrier per slot; page-table entries are read one unit before they are
// needed.  Every warp keeps its own online-softmax state; a pair that spans
// several warps is merged through shared memory, a pair that spans several
// CTAs through a partial in the workspace merged by the CTA that finishes it
// last (an atomic ticket per pair, reset by that CTA).  Every mbarrier wait is
// bounded.
#pragma once

#include <cuda.h>
#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_tc_ptx.cuh"
#include "kvq_mma_ptx.cuh"

namespace kvq {
namespace mma {

using namespace ptx;

constexpr int D = 128;
constexpr int NKG = 4;                         // key groups of 32 channels
constexpr int kMaxWarps = 8;
constexpr int kMaxSpw = 4;                     // ring slots per warp
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
    static constexpr int UP = 1;                         // pages per quantized unit
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
    // slots start 1024-byte aligned (the window tiles use the 128-byte TMA swizzle)
    static constexpr int SLOT = ((QBYTES > 2 * WROWS ? QBYTES : 2 * WROWS) + 1023) & ~1023;
    // eight warps when two slots each fit beside the per-warp areas, else four
    static constexpr int NW = 8 * 2 * SLOT <= 160 * 1024 ? 8 : 4;
    static constexpr int QAREA = NH * 512 + NH * 32;     // per warp: limb / bf16 query staging + scalars
    static_assert(KCODES % 16 == 0 && KMETA % 16 == 0 && VCODES % 16 == 0 && VMETA % 16 == 0, "bulk sizes");
};

struct Head {
    uint64_t full[kMaxWarps][kMaxSpw];
    int upg[kMaxWarps][kMaxSpw];           // page of the unit in each slot (-1: none)
    int cnt[kMaxWarps][2];                 // warps done with a pair they share, by owner warp and kind
    int wfirst[kMaxWarps], wlast[kMaxWarps];   // pairs of each warp's first and last unit (-1: no units)
    int abort;
    int done;                              // warps past their units
};

// merge partials: per head a row of D outputs, the running maximum and the
// weight sum, padded to PST floats so that every row starts 16-byte aligned
constexpr int PST = D + 4;
template <int NH>
__host__ __device__ constexpr int part_floats() { return NH * PST; }

__host__ __device__ inline int off_sched() { return (int(sizeof(Head)) + 15) & ~15; }
__host__ __device__ inline int off_qarea(int batch) { return (off_sched() + 8 * (batch + 1) + 127) & ~127; }
// a warp's first segment, when another warp began its pair, is parked here
// until the merge: one partial of g heads per warp
template <int KB, int VB, int NH>
__host__ __device__ inline int off_park(int batch) {
    return (off_qarea(batch) + Cfg<KB, VB, NH>::NW * Cfg<KB, VB, NH>::QAREA + 127) & ~127;
}
// (the ring itself starts at the next 1024-byte aligned address from here)
template <int KB, int VB, int NH>
__host__ __device__ inline int off_ring(int batch, int g) {
    return (off_park<KB, VB, NH>(batch) + Cfg<KB, VB, NH>::NW * NH * PST * 4 + 127) & ~127;
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

// Window rows arrive as TMA tiles of 16 rows x 64 channels (128 bytes) with
// the 128-byte swizzle: in tile row r the 16-byte chunk c sits at position
// c ^ (r mod 8), so the eight rows an ldmatrix reads (tokens r .. r+7 at one
// chunk) fall in eight distinct bank groups.  Tiles of the key (or value)
// rows of a unit: [16-row block][channel half] of 2 KB each.
__device__ __forceinline__ uint32_t wrow(uint32_t base, int t, int c) {
    const int tt = t & 15;
    return base + (t >> 4) * 4096 + (c >> 3) * 2048 + tt * 128 + (((c & 7) ^ (tt & 7)) << 4);
}
// 2-D tiled TMA load (no multicast) of the box at (x, y) into shared memory
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------- schedule
struct UnitPos {
    int b, h, j, n;
    int L, nq;      // the sequence's length and quantized units (set per pair)
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
    return {lo, r / n, r % n, n, 0, 0};
}

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

// The query of kv-head h of sequence b: lane l gets channels 4l .. 4l+3 of
// each of the NH heads (zeros for heads r >= g).  All loads are issued before
// any is used.
template <int NH>
__device__ __forceinline__ void load_query(const Params& p, const void* q, int q_bf16, int b, int h, int lane,
                                           float (&x)[NH][4]) {
    const int g = p.g;
    const size_t row0 = (size_t(b) * p.hq + size_t(h) * g) * D + 4 * lane;
    if (q_bf16) {
        uint2 v[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r)
            v[r] = r < g ? __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(q) + row0 +
                                                                 size_t(r) * D))
                         : make_uint2(0u, 0u);
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            x[r][0] = bf_lo(v[r].x);
            x[r][1] = bf_hi(v[r].x);
            x[r][2] = bf_lo(v[r].y);
            x[r][3] = bf_hi(v[r].y);
        }
    } else {
        float4 v[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r)
            v[r] = r < g ? __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(q) + row0 + size_t(r) * D))
                         : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            x[r][0] = v[r].x;
            x[r][1] = v[r].y;
            x[r][2] = v[r].z;
            x[r][3] = v[r].w;
        }
    }
}

// ---------------------------------------------------------------- query preparation
// Query of kv-head h of sequence b: int8 limbs of the (rotated) query in the
// score MMA's K order, staged in the warp's area, then read into the B
// fragments; per head the limb unit (times sm_scale*log2 e) and the sums of
// the rotated query per key group (times the same).
template <int KB, int NH>
__device__ __forceinline__ void prep_query(const Params& p, const float (&xq)[NH][4], uint8_t* qa, float sl2, int lane,
                           uint32_t (&qb)[NKG][Cfg<KB, 1, NH>::NT][2], float (&cq)[NH / 4],
                           float (&cz)[NH / 4][NKG]) {
    constexpr int NT = Cfg<KB, 1, NH>::NT;
    const int g = p.g;
    int8_t* ql = reinterpret_cast<int8_t*>(qa);                 // [limb][head][group][32]
    float* qs = reinterpret_cast<float*>(qa + NH * 512);         // [head][8]
#pragma unroll 1
    for (int r = 0; r < NH; ++r) {
        float x[4] = {xq[r][0], xq[r][1], xq[r][2], xq[r][3]};
        if (r < g && p.rotate) rotate_warp<D>(x, p.signs, lane);
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
__device__ __forceinline__ void prep_window_query(const Params& p, const void* q, int q_bf16, int b, int h, uint8_t* qa, int lane) {
    __nv_bfloat16* wq = reinterpret_cast<__nv_bfloat16*>(qa);
    float xq[NH][4];
    load_query<NH>(p, q, q_bf16, b, h, lane, xq);
    __syncwarp();
#pragma unroll
    for (int r = 0; r < NH; ++r) {
        const float* x = xq[r];
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

// ---------------------------------------------------------------- end of a segment
// What the end of a segment reads besides the warp's accumulators.
struct Split {
    int U, NC;              // units, CTAs with units (NC <= U)
    int q, r;               // U = q NC + r
    float inv_nc, inv_u;    // 1 / NC, NC / U
};
__device__ __forceinline__ Split make_split(int U, int NC) {
    return {U, NC, U / NC, U % NC, 1.0f / float(NC), float(NC) / float(U)};
}
// floor(t / NC) for 0 <= t < 2^24, from the float quotient corrected by one step
__device__ __forceinline__ int div_nc(int t, const Split& s) {
    int d = int(float(t) * s.inv_nc);
    if ((d + 1) * s.NC <= t) ++d;
    if (d * s.NC > t) --d;
    return d;
}
// first unit of CTA c: floor(c U / NC) = c q + floor(c r / NC)
__device__ __forceinline__ int cta_start(int c, const Split& s) { return c * s.q + div_nc(c * s.r, s); }
// CTA holding unit u
__device__ __forceinline__ int cta_of(int u, const Split& s) {
    int c = min(s.NC - 1, int(float(u) * s.inv_u));
    while (c + 1 < s.NC && cta_start(c + 1, s) <= u) ++c;
    while (c > 0 && cta_start(c, s) > u) --c;
    return c;
}

struct SegCtx {
    Head* hd;
    const int* S;           // units per pair, prefix over sequences
    float* park;            // [NW][NH][PST] parked first segments
    uint8_t* ring;          // the warps' rings (a warp's final partial goes to its first slot)
    float* out;
    float* lse;
    float* part;            // [CTAs][2][NH][PST] partials of pairs split between CTAs
    uint32_t* tickets;
    unsigned* status;
    int hq, g, H, SPW, slot_bytes, cs, ce, base_n, rem;
    Split sp;
};

// normalized output and lse of heads tig (+4) of kv-head h of sequence b
template <int NH>
__device__ __forceinline__ void write_final(const SegCtx& c, const State<NH>& x, int b, int h, int lane) {
    const int g8 = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int hs = 0; hs < NH / 4; ++hs) {
        const float lt = grp_sum(x.l[hs]), zt = grp_sum(x.pz[hs]);
        const int r = tig + 4 * hs;
        if (r >= c.g) continue;
        const size_t row = size_t(b) * c.hq + size_t(h) * c.g + r;
        const float inv = lt > 0.0f ? 1.0f / lt : 0.0f;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            c.out[row * D + 16 * mt + g8] = x.bad ? NAN : (x.o[hs][mt][0] + zt) * inv;
            c.out[row * D + 16 * mt + g8 + 8] = x.bad ? NAN : (x.o[hs][mt][1] + zt) * inv;
        }
        if (c.lse && g8 == 0)
            c.lse[row] = x.bad ? NAN : (lt > 0.0f ? (x.m[hs] + log2f(lt)) * kLn2 : -INFINITY);
    }
}

// unnormalized partial: per head D outputs (including the zero-point term),
// the running maximum (log2 domain) and the weight sum
template <int NH>
__device__ __forceinline__ void store_partial(const SegCtx& c, const State<NH>& x, float* dst, int lane) {
    const int g8 = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int hs = 0; hs < NH / 4; ++hs) {
        const float lt = grp_sum(x.l[hs]), zt = grp_sum(x.pz[hs]);
        const int r = tig + 4 * hs;
        if (r >= c.g) continue;
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
}

__device__ __forceinline__ float4 ld_relaxed_v4(const float* a) {
    float4 v;
    asm volatile("ld.relaxed.gpu.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(a)
                 : "memory");
    return v;
}
__device__ __forceinline__ float2 ld_relaxed_v2(const float* a) {
    float2 v;
    asm volatile("ld.relaxed.gpu.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(a) : "memory");
    return v;
}

// Merge the partials of pair P: first those of warps wlo .. whi of this CTA
// (parked first segments, or final segments in the warps' rings); a pair
// inside the CTA is then output.  For a pair split between CTAs every CTA
// stores its merged partial and then takes a ticket of the pair; the CTA that
// takes the last ticket merges every CTA's partial in CTA order (the result
// does not depend on the order the CTAs finished in), outputs and resets the
// ticket, so that no CTA waits for another.  One loop over all the partials
// keeps the code short (it runs cold, once or twice per warp).
// Lane l owns channels 4l .. 4l+3.
template <int NH>
__device__ __forceinline__ void merge_pair(const SegCtx& c, int P, int wlo, int whi, int lane, bool dry = false) {
    const int g = c.g, H = c.H;
    const int b = P / H, h = P - b * H;
    const int n = c.S[b + 1] - c.S[b];
    const int u0 = H * c.S[b] + h * n, u1 = u0 + n;
    const bool inside = u0 >= c.cs && u1 <= c.ce;
    const int cta = blockIdx.x;
    float M[NH], Ls[NH], O[NH][4];
    auto reset = [&](float l0) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            M[r] = -INFINITY;
            Ls[r] = l0;
            O[r][0] = O[r][1] = O[r][2] = O[r][3] = 0.0f;
        }
    };
    // every row of a partial is loaded before any is folded (a slot always holds
    // NH rows; those of heads r >= g are read and ignored): parts of this CTA
    // from shared memory with plain loads (the counter's acquire orders them),
    // other CTAs' partials with relaxed loads at GPU scope (past the L1)
    auto load_local = [&](const float* src, float2 (&ml)[NH], float4 (&v)[NH]) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            ml[r] = *reinterpret_cast<const float2*>(src + r * PST + D);
            v[r] = *reinterpret_cast<const float4*>(src + r * PST + 4 * lane);
        }
    };
    auto load = [&](const float* src, float2 (&ml)[NH], float4 (&v)[NH]) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            ml[r] = ld_relaxed_v2(src + r * PST + D);
            v[r] = ld_relaxed_v4(src + r * PST + 4 * lane);
        }
    };
    auto fold = [&](const float2 (&ml)[NH], const float4 (&v)[NH]) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            if (r >= g) continue;
            const float mn = fmaxf(M[r], ml[r].x);
            const float mu = mn == -INFINITY ? 0.0f : mn;
            const float al = M[r] == -INFINITY ? 0.0f : ex2(M[r] - mu);
            const float wgt = ml[r].x == -INFINITY ? 0.0f : ex2(ml[r].x - mu);
            M[r] = mn;
            Ls[r] = fmaf(ml[r].y, wgt, Ls[r] * al);
            O[r][0] = fmaf(v[r].x, wgt, O[r][0] * al);
            O[r][1] = fmaf(v[r].y, wgt, O[r][1] * al);
            O[r][2] = fmaf(v[r].z, wgt, O[r][2] * al);
            O[r][3] = fmaf(v[r].w, wgt, O[r][3] * al);
        }
    };
    reset(0.0f);
    // the parts of this CTA's warps
#pragma unroll 1
    for (int ww = wlo; ww <= whi; ++ww) {
        const bool parked = c.hd->wfirst[ww] == P && c.hd->wlast[ww] != P;
        float2 ml[NH];
        float4 v[NH];
        load_local(parked ? c.park + ww * NH * PST
                          : reinterpret_cast<const float*>(c.ring + size_t(ww) * c.SPW * c.slot_bytes),
                   ml, v);
        fold(ml, v);
    }
    if (!inside) {
        const int ca = cta_of(u0, c.sp), cb = cta_of(u1 - 1, c.sp);
        // this CTA's partial goes to its slot (0 when P is the CTA's first pair, else 1)
        float* gdst = c.part + (size_t(cta) * 2 + (u0 > c.cs ? 1 : 0)) * part_floats<NH>();
        if (!dry) {
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                if (r >= g) continue;
                *reinterpret_cast<float4*>(gdst + r * PST + 4 * lane) = make_float4(O[r][0], O[r][1], O[r][2], O[r][3]);
                if (lane == 0) *reinterpret_cast<float2*>(gdst + r * PST + D) = make_float2(M[r], Ls[r]);
            }
        }
        __syncwarp();                         // every lane's stores, then lane 0's release
        const unsigned need = unsigned(cb - ca);   // tickets taken before the last one
        unsigned old = need;
        if (lane == 0 && !dry) old = atom_add_acq_rel_gpu(c.tickets + P, 1u);
        old = __shfl_sync(FULL, old, 0);
        if (old < need) return;
        // the last CTA folds every CTA's partial, its own too, in CTA order, so that
        // the result does not depend on which CTA finished last; two at a time
        const bool bad = old > need;          // the ticket was not zero at the start of the call
        if (bad && lane == 0) atomicAdd(&c.status[1], 1u);
        reset(bad ? NAN : 0.0f);
        __syncwarp();                         // lane 0's acquire, then every lane's loads
#pragma unroll 1
        for (int cc = ca; cc <= cb; cc += 2) {
            const bool two = cc + 1 <= cb;
            const float* s0 = c.part + (size_t(cc) * 2 + (u0 > cta_start(cc, c.sp) ? 1 : 0)) * part_floats<NH>();
            const float* s1 = two ? c.part + (size_t(cc + 1) * 2 + (u0 > cta_start(cc + 1, c.sp) ? 1 : 0)) * part_floats<NH>()
                                  : s0;
            float2 ml0[NH], ml1[NH];
            float4 v0[NH], v1[NH];
            load(s0, ml0, v0);
            load(s1, ml1, v1);
            fold(ml0, v0);
            if (two) fold(ml1, v1);
        }
        if (lane == 0 && !dry) c.tickets[P] = 0u;   // ready for the next call
    }
    // lane r < g: the reciprocal weight sum and the lse of head r
    float myL = Ls[0], myM = M[0];
#pragma unroll
    for (int r = 1; r < NH; ++r)
        if (lane == r) myL = Ls[r], myM = M[r];
    const float inv = myL > 0.0f ? __fdividef(1.0f, myL) : 0.0f;   // within 2 ulp
    const size_t row0 = size_t(b) * c.hq + size_t(h) * g;
    const float lv = myL > 0.0f ? (myM + log2f(myL)) * kLn2 : (myL == 0.0f ? -INFINITY : NAN);
    if (c.lse && lane < g && !dry) c.lse[row0 + lane] = lv;
#pragma unroll
    for (int r = 0; r < NH; ++r) {
        const float ir = __shfl_sync(FULL, inv, r);
        if (r < g && !dry)
            *reinterpret_cast<float4*>(c.out + (row0 + r) * D + 4 * lane) =
                make_float4(O[r][0] * ir, O[r][1] * ir, O[r][2] * ir, O[r][3] * ir);
    }
}

// The segment of warp w that ends here covers part of kv-head h of sequence b,
// shared with other warps or CTAs: the partial is stored (the warp's first
// segment to its parking area, its final one to its ring, whose copies are all
// consumed) and counted.  Returns the pair when this warp was the last of the
// CTA's warps that hold a part of it (it then owes the merge of warps
// wlo .. whi, done after its units, so that the merge code runs once per warp
// at most twice and never between two units), else -1.
template <int NH>
__device__ __forceinline__ int post_segment(const SegCtx& c, const State<NH>& x, int b, int h, bool last_unit, int w,
                                            int lane, int& wlo, int& whi) {
    store_partial<NH>(c, x, last_unit ? reinterpret_cast<float*>(c.ring + size_t(w) * c.SPW * c.slot_bytes)
                                      : c.park + w * NH * PST, lane);
    const int P = b * c.H + h, n = c.S[b + 1] - c.S[b];
    const int u0 = c.H * c.S[b] + h * n, u1 = u0 + n;
    // warp holding unit u of this CTA's range
    auto warp_of = [&](int u) -> int {
        const int x0 = u - c.cs, big = c.rem * (c.base_n + 1);
        return x0 < big ? x0 / (c.base_n + 1) : c.rem + (x0 - big) / c.base_n;
    };
    wlo = warp_of(u0 > c.cs ? u0 : c.cs);
    whi = warp_of((u1 < c.ce ? u1 : c.ce) - 1);
    const int kind = c.hd->wlast[wlo] == P ? 1 : 0;
    __syncwarp();                             // every lane's stores, then lane 0's release
    int old = 0;
    if (lane == 0) old = atom_add_acq_rel_cta(&c.hd->cnt[wlo][kind], 1);
    old = __shfl_sync(FULL, old, 0);
    return old == whi - wlo ? P : -1;
}

// ---------------------------------------------------------------- the kernel
template <int KB, int VB, int NH>
__global__ void __launch_bounds__(Cfg<KB, VB, NH>::NW * 32, 1)
decode_mma_kernel(const __grid_constant__ Params p, const void* __restrict__ q, const int q_bf16, const int32_t* __restrict__ lens,
                  const int max_len, const float sl2, float* __restrict__ out, float* __restrict__ lse,
                  float* __restrict__ part, uint32_t* __restrict__ tickets, const int SPW, const int after_append,
                  unsigned int* __restrict__ status, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v) {
    using C = Cfg<KB, VB, NH>;
    constexpr int HS = C::HS, NT = C::NT, TOK = C::TOK, WU = C::WU, NW = C::NW, kThreads = NW * 32;
    extern __shared__ __align__(1024) uint8_t smem[];
    Head& hd = *reinterpret_cast<Head*>(smem);
    const int B = p.batch, H = p.hkv, g = p.g;
    int* S = reinterpret_cast<int*>(smem + off_sched());    // [B+1] units of one pair of sequences < b
    int* LB = S + (B + 1);                                    // [B] clamped lengths  (S, LB: 8(B+1) bytes)
    uint8_t* qarea = smem + off_qarea(B);
    float* park = reinterpret_cast<float*>(smem + off_park<KB, VB, NH>(B));   // [NW][NH][PST]
    uint8_t* ring;                                                          // [NW][SPW][SLOT], 1024-aligned
    {
        const uint32_t a = smem_u32(smem) + off_ring<KB, VB, NH>(B, p.g);
        ring = smem + (((a + 1023u) & ~1023u) - smem_u32(smem));
    }
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
        for (int w = 0; w < NW; ++w)
            for (int i = 0; i < SPW; ++i) mbar_init(&hd.full[w][i], 1);
        mbar_fence_init();
        hd.abort = 0;
        hd.done = 0;
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
    const int U = H * S[B], NC = min(int(gridDim.x), U);
    const Split sp = make_split(U, NC);
    const int cta = blockIdx.x;
    const int cs = cta < NC ? cta_start(cta, sp) : 0, ce = cta < NC ? cta_start(cta + 1, sp) : 0;
    const int len = ce - cs, base_n = len / NW, rem = len % NW;
    if (tid < NW * 2) hd.cnt[tid >> 1][tid & 1] = 0;
    if (tid < NW) {
        const int n = base_n + (tid < rem ? 1 : 0), u0 = cs + tid * base_n + min(tid, rem);
        int pf = -1, pl = -1;
        if (n > 0) {
            const UnitPos a = locate(S, B, H, u0), z = locate(S, B, H, u0 + n - 1);
            pf = a.b * H + a.h;
            pl = z.b * H + z.h;
        }
        hd.wfirst[tid] = pf;
        hd.wlast[tid] = pl;
    }
    __syncthreads();
    if (len <= 0) return;

    const int w = warp, g8 = lane >> 2, tig = lane & 3;
    const int nunits = base_n + (w < rem ? 1 : 0);
    const int wbeg = cs + w * base_n + min(w, rem);
    uint8_t* qa = qarea + w * C::QAREA;
    uint8_t* wring = ring + size_t(w) * SPW * C::SLOT;
    const uint32_t wring_s = smem_u32(wring);
    auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&hd.abort) != 0; };
    // warp-collective bounded wait: every lane gets the same answer
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
        bool ok = !aborted() && mbar_wait(bar, parity, kWaitNs);
        ok = __all_sync(FULL, ok);
        if (!ok && lane == 0 && atomicExch(&hd.abort, 1) == 0) atomicAdd(&status[0], 1u);
        return ok;
    };
    // page-table entry of unit u when it is a quantized unit, else -1; the
    // value is checked where it is used, so that the load is not waited for here
    auto page_raw = [&](const UnitPos& u) -> int {
        const int L = LB[u.b], lq = L - min(W, L), nq = (lq + TOK - 1) / TOK;
        int v = -1;
        if (L > 0 && u.j < nq && u.j < p.max_pages) v = __ldg(p.page_table + size_t(u.b) * p.max_pages + u.j);
        return v;
    };
    // length and quantized units of the unit's sequence (kept per pair)
    auto fill = [&](UnitPos& u) {
        u.L = LB[u.b];
        u.nq = (u.L - min(W, u.L) + TOK - 1) / TOK;
    };
    auto next_unit = [&](UnitPos& u) {
        if (++u.j == u.n) {
            u.j = 0;
            if (++u.h == H) {
                u.h = 0;
                if (u.b + 1 < B) ++u.b;
            }
            u.n = S[u.b + 1] - S[u.b];
            fill(u);
        }
    };
    int issued = 0;                     // units whose copies this warp has issued
    // page-table entries of this warp's units: lane l holds those of units l, l+32, l+64, l+96
    int pgr[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) pgr[r] = lane + 32 * r < nunits ? page_raw(locate(S, B, H, wbeg + lane + 32 * r)) : -1;
    // copies of unit u (the warp's unit k) into this warp's slot `slot`
    auto issue = [&](int slot, const UnitPos& u, int k) {
        int raw;
        if (k < 128) {
            const int v = k < 32 ? pgr[0] : (k < 64 ? pgr[1] : (k < 96 ? pgr[2] : pgr[3]));
            raw = __shfl_sync(FULL, v, k & 31);
        } else {
            raw = page_raw(u);
        }
        ++issued;
        const int pg = (raw >= 0 && raw < p.num_pages) ? raw : -1;
        if (lane == 0) hd.upg[w][slot] = pg;
        uint64_t* bar = &hd.full[w][slot];
        uint8_t* sl = wring + size_t(slot) * C::SLOT;
        const int L = u.L, nq = u.nq;
        if (L > 0 && u.j < nq) {
            // a page: the four blocks in 16-byte pieces from every lane (a bulk copy
            // holds the lane that issues it for about a hundred cycles, so four of
            // them per unit cost more than these); each lane's copies arrive on the
            // slot's barrier when they land, lane 0 adds the barrier's one arrival
            if (pg >= 0) {
                const size_t blk = size_t(pg) * H + u.h;
                const uint32_t s0 = smem_u32(sl);
                const uint8_t* kc = p.k_codes + blk * C::KCODES;
                const uint8_t* km = reinterpret_cast<const uint8_t*>(p.k_meta + blk * (kPage * NKG));
                const uint8_t* vc = p.v_codes + blk * C::VCODES;
                const uint8_t* vm = reinterpret_cast<const uint8_t*>(p.v_meta + blk * kPage);
#pragma unroll
                for (int i = lane; i < C::KCODES / 16; i += 32) cp16(s0 + 16 * i, kc + 16 * i);
#pragma unroll
                for (int i = lane; i < C::KMETA / 16; i += 32) cp16(s0 + C::OFF_KM + 16 * i, km + 16 * i);
#pragma unroll
                for (int i = lane; i < C::VCODES / 16; i += 32) cp16(s0 + C::OFF_VC + 16 * i, vc + 16 * i);
#pragma unroll
                for (int i = lane; i < C::VMETA / 16; i += 32) cp16(s0 + C::OFF_VM + 16 * i, vm + 16 * i);
                cp_async_arrive(bar);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_plain(bar);
        } else if (L > 0) {
            // window unit: ring slots [(j - nq) * WU, + WU) of the pair, whose rows are
            // contiguous (the window's positions fill ring slots [0, min(W, L)); the
            // order of positions does not matter to attention).  Keys then values, as
            // 16-row x 64-channel TMA tiles.
            const int y0 = (u.b * H + u.h) * W + (u.j - nq) * WU;
            fence_proxy_async();        // every lane's earlier writes to the slot (cp.async pieces) first
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, uint32_t(2 * WU * D * 2));
                const uint32_t s0 = smem_u32(sl);
#pragma unroll
                for (int rb = 0; rb < WU / 16; ++rb)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        tma_load_2d(s0 + rb * 4096 + half * 2048, &tm_k, half * 64, y0 + rb * 16, bar);
                        tma_load_2d(s0 + C::WROWS + rb * 4096 + half * 2048, &tm_v, half * 64, y0 + rb * 16, bar);
                    }
            }
            __syncwarp();
        } else {
            if (lane == 0) mbar_arrive_plain(bar);
        }
    };

    State<NH> st;
    st.reset();

    if (nunits > 0) {
        // ---- the first pair's query (loaded before the copies so that its loads
        // are not queued behind them), then the first SPW units: page lookups in
        // parallel, then the copies
        UnitPos pos = locate(S, B, H, wbeg);
        fill(pos);
        UnitPos ip = pos;
        float xq[NH][4];
        load_query<NH>(p, q, q_bf16, pos.b, pos.h, lane, xq);
        int seg_j0 = pos.j;
        uint32_t qb[NKG][NT][2];
        float cq[HS], cz[HS][NKG];
        bool q_ready = false, wq_ready = false;
        if (after_append) {
            // launched as the programmatic dependent of an append on the same stream:
            // everything so far read only what the append does not write (lengths,
            // page table, query), so the query is prepared too before the wait for
            // the append's results; the cache is read only after it
            prep_query<KB, NH>(p, xq, qa, sl2, lane, qb, cq, cz);
            q_ready = true;
            asm volatile("griddepcontrol.wait;" ::: "memory");
        }
        for (int i = 0; i < SPW && i < nunits; ++i) {
            issue(i, ip, i);
            next_unit(ip);
        }
        int mp0 = -1, mlo0 = 0, mhi0 = 0, mp1 = -1, mlo1 = 0, mhi1 = 0;   // merges this warp owes
        int slot = 0;
        uint32_t phase = 0;             // parity of the slot's barrier for this unit
        for (int k = 0; k < nunits; ++k) {
            // the pair's query (one place for the first pair and every later one)
            if (!q_ready) {
                if (k > 0) load_query<NH>(p, q, q_bf16, pos.b, pos.h, lane, xq);
                prep_query<KB, NH>(p, xq, qa, sl2, lane, qb, cq, cz);
                q_ready = true;
            }
            const int L = pos.L, wl = min(W, L), lq = L - wl, nq = pos.nq;
            const uint32_t sl = wring_s + uint32_t(slot) * C::SLOT;
            const bool kind_q = L > 0 && pos.j < nq;
            const bool kind_w = L > 0 && pos.j >= nq;
            const int pres1 = 0;
            if (kind_w && !wq_ready) {
                prep_window_query<NH>(p, q, q_bf16, pos.b, pos.h, qa, lane);
                wq_ready = true;
            }
            const bool ok = wait_bar(&hd.full[w][slot], phase);
            if (!ok) st.bad = true;
            const int pres0 = kind_q && hd.upg[w][slot] >= 0;
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
                                for (int nt = 0; nt < NT; ++nt) mma_u8s8_z(d[nt], a, qb[grp][nt][0], qb[grp][nt][1]);
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
                        for (int s4 = 0; s4 < 2 * C::UP; ++s4) {
                            uint32_t a[4];
                            vfrag<VB>(sl + C::OFF_VC + (s4 >> 1) * C::VCODES, chA, chB, s4 & 1, tig, a);
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                if (s4 == 0) mma_u8u8_z(acc[nt], a, bq[s4][nt][0], bq[s4][nt][1]);
                                else mma_u8u8(acc[nt], a, bq[s4][nt][0], bq[s4][nt][1]);
                            }
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
                    const int cnt = min(WU, wl - (pos.j - nq) * WU);    // ring slots of the unit that hold tokens
                    const __nv_bfloat16* wq = reinterpret_cast<const __nv_bfloat16*>(qa);
                    const uint32_t kbase = sl, vbase = sl + C::WROWS;
                    if (cnt < WU) {
                        // value rows past the window's end: zeros, so that their zero weights
                        // meet finite values in the ·V product
                        for (int idx = lane; idx < (WU - cnt) * 16; idx += 32)
                            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(wrow(vbase, cnt + (idx >> 4), idx & 15)),
                                         "r"(0)
                                         : "memory");
                        fence_proxy_async();    // before a later bulk copy into this slot
                        __syncwarp();
                    }
                    float sw[HS][NB][2];
#pragma unroll
                    for (int bb = 0; bb < NB; ++bb) {
                        float d[HS][4];
                        const int mi = lane >> 3, r = lane & 7;
                        const int tq = 16 * bb + r + 8 * (mi & 1);      // score rows: tokens in order
#pragma unroll
                        for (int s8 = 0; s8 < 8; ++s8) {
                            uint32_t a[4];
                            ldsm_x4(a, wrow(kbase, tq, 2 * s8 + (mi >> 1)));
#pragma unroll
                            for (int hs = 0; hs < HS; ++hs) {
                                const int head = (g8 >> 1) + 4 * hs, hl = g8 & 1;
                                const __nv_bfloat16* qq = wq + (head * 2 + hl) * D + 16 * s8 + 2 * tig;
                                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(qq);
                                const uint32_t b1 = *reinterpret_cast<const uint32_t*>(qq + 8);
                                if (s8 == 0) mma_bf16_z(d[hs], a, b0, b1);
                                else mma_bf16(d[hs], a, b0, b1);
                            }
                        }
                        const int t0 = 16 * bb + g8;                   // rows g8 and g8 + 8
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs) {
                            sw[hs][bb][0] = t0 < cnt ? (d[hs][0] + d[hs][1]) * sl2 : -INFINITY;
                            sw[hs][bb][1] = t0 + 8 < cnt ? (d[hs][2] + d[hs][3]) * sl2 : -INFINITY;
                        }
                    }
                    float alpha[HS];
                    uint32_t px[HS][NB][2];          // per row (g8, g8 + 8): bf16 {high, low} of p
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
                            const uint32_t hi = pack_bf16(p0, p1);
                            const uint32_t lo = pack_bf16(p0 - bf_lo(hi), p1 - bf_hi(hi));
                            px[hs][bb][0] = __byte_perm(hi, lo, 0x5410);   // row g8:     {high, low}
                            px[hs][bb][1] = __byte_perm(hi, lo, 0x7632);   // row g8 + 8: {high, low}
                        }
                        st.l[hs] = fmaf(st.l[hs], alpha[hs], ls);
                        st.pz[hs] *= alpha[hs];
                    }
                    // B fragment of the weights: tokens 2tig, 2tig+1 (and 8 more) of column
                    // (head g8/2, high or low part g8%2), held by the lanes of rows 2tig, 2tig+1
                    uint32_t bv[NB][HS][2];
                    const int se = 4 * (2 * tig) + (g8 >> 1), so = se + 4;
                    const uint32_t sel = (g8 & 1) ? 0x7632u : 0x5410u;
#pragma unroll
                    for (int bb = 0; bb < NB; ++bb)
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs)
#pragma unroll
                            for (int hf = 0; hf < 2; ++hf) {
                                const uint32_t xe = __shfl_sync(FULL, px[hs][bb][hf], se);
                                const uint32_t xo = __shfl_sync(FULL, px[hs][bb][hf], so);
                                bv[bb][hs][hf] = __byte_perm(xe, xo, sel);
                            }
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        float dv[HS][4];
                        const int mi = lane >> 3, r = lane & 7;
#pragma unroll
                        for (int bb = 0; bb < NB; ++bb) {
                            uint32_t a[4];
                            ldsm_x4_t(a, wrow(vbase, 16 * bb + r + 8 * (mi >> 1), 2 * mt + (mi & 1)));
#pragma unroll
                            for (int hs = 0; hs < HS; ++hs) {
                                if (bb == 0) mma_bf16_z(dv[hs], a, bv[bb][hs][0], bv[bb][hs][1]);
                                else mma_bf16(dv[hs], a, bv[bb][hs][0], bv[bb][hs][1]);
                            }
                        }
#pragma unroll
                        for (int hs = 0; hs < HS; ++hs) {
                            st.o[hs][mt][0] = fmaf(st.o[hs][mt][0], alpha[hs], dv[hs][0] + dv[hs][1]);
                            st.o[hs][mt][1] = fmaf(st.o[hs][mt][1], alpha[hs], dv[hs][2] + dv[hs][3]);
                        }
                    }
                }
                __syncwarp();
                // ---- the slot is free: copies of unit k + SPW into it
                if (k + SPW < nunits && ok) {
                    issue(slot, ip, k + SPW);
                    next_unit(ip);
                }

                // ---- end of a segment: the pair is done, or the warp's range ends
                const bool pair_end = pos.j + 1 == pos.n, last_unit = k + 1 == nunits;
                if (pair_end || last_unit) {
                    const SegCtx sc{&hd, S, park, ring, out, lse, part, tickets, status, p.hq, g, H, SPW, C::SLOT,
                                    cs, ce, base_n, rem, sp};
                    if (seg_j0 == 0 && pair_end) {    // the whole pair in this warp: final output
                        write_final<NH>(sc, st, pos.b, pos.h, lane);
                    } else {
                        int lo, hi;
                        const int P = post_segment<NH>(sc, st, pos.b, pos.h, last_unit, w, lane, lo, hi);
                        if (P >= 0) {
                            if (mp0 < 0) {
                                mp0 = P, mlo0 = lo, mhi0 = hi;
                            } else {
                                mp1 = P, mlo1 = lo, mhi1 = hi;
                            }
                        }
                    }
                    st.reset();
                }
                // ---- next unit
                if (++slot == SPW) {
                    slot = 0;
                    phase ^= 1u;
                }
                if (!pair_end) {
                    ++pos.j;
                } else if (!last_unit) {
                    pos.j = 0;
                    if (++pos.h == H) {
                        pos.h = 0;
                        ++pos.b;
                    }
                    pos.n = S[pos.b + 1] - S[pos.b];
                    fill(pos);
                    seg_j0 = 0;
                    q_ready = wq_ready = false;
                }
            }

        // ---- the merges this warp owes (the partials stay where they were stored:
        // parking areas and the rings of warps that are done with their units).
        // A warp that owes none and is among the first half of the CTA's warps to
        // be done runs the merge code once without effects (no stores, no
        // tickets; loads from the CTA's first pair's parts), so that the merging
        // warps of this SM find that code in the instruction cache.
        int rank_done = 0;
        if (lane == 0) rank_done = atomicAdd(&hd.done, 1);
        rank_done = __shfl_sync(FULL, rank_done, 0);
        if (mp0 < 0 && rank_done < NW / 2) {
            const SegCtx sc{&hd, S, park, ring, out, lse, part, tickets, status, p.hq, g, H, SPW, C::SLOT,
                            cs, ce, base_n, rem, sp};
            const UnitPos f = locate(S, B, H, cs);
            merge_pair<NH>(sc, f.b * H + f.h, 0, 0, lane, true);
        }
        if (mp0 >= 0) {
            const SegCtx sc{&hd, S, park, ring, out, lse, part, tickets, status, p.hq, g, H, SPW, C::SLOT,
                            cs, ce, base_n, rem, sp};
#pragma unroll 1
            for (int i = 0; i < 2; ++i) {
                const int P = i ? mp1 : mp0;
                if (P >= 0) merge_pair<NH>(sc, P, i ? mlo1 : mlo0, i ? mhi1 : mhi0, lane);
            }
        }

        if (aborted()) {
            // nothing may still be copying into shared memory when the CTA exits
            for (int u = max(0, issued - SPW); u < issued; ++u) mbar_wait(&hd.full[w][u % SPW], (u / SPW) & 1, kDrainNs);
        }
    }

}

}  // namespace mma
}  // namespace kvq

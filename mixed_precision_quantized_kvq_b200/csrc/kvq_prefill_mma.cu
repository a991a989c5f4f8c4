// Chunked-prefill attention over the quantized cache on the tensor cores
// (mma.sync, bf16 operands, fp32 accumulation) for head_dim 128, key groups
// of 32 channels of one token and unrotated keys.
//
// What it computes is what the CUDA-core body (kvq_prefill_body.cuh) computes
// ("Kuantisasi KV cache mengganggu attention ...", sections "Error pada key
// masuk sebelum softmax" and "Pertumbuhan cache mengubah trade pada
// serving"): query i of a chunk of n attends causally to positions
// [0, L-n+i], pages reconstructed as code*scale + zero in fp32 below L-W and
// the bf16 window above.
//
// One CTA takes 128 (query, head) rows of one (sequence, kv-head): 128/g
// queries with the g heads of the kv-group; each of its 8 warps owns 16 rows.
// Per 64-position tile the CTA reconstructs keys and values once into shared
// memory, each value x as a bf16 pair (hi = bf16(x), lo = bf16(x - hi)), and
// every warp runs its rows through it in registers, flash-attention style:
//   S = Q K^T  as  Qh Kh + Qh Kl + Ql Kh   (mma m16n8k16, three products),
//   online softmax of S (log2 domain) in registers,
//   O += P V   as  Ph Vh + Ph Vl + Pl Vh,
// with the score accumulators reused as the A fragments of P.  The dropped
// lo*lo products and the bf16 splits leave about 2^-16 relative error per
// product, far inside the 1e-3 tolerance.  Keys are stored [position][channel]
// and values [channel][position] (the B operands' k-contiguous order), in
// 16-byte chunks swizzled by row so that ldmatrix reads hit 8 distinct bank
// groups.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.cuh"
#include "kvq_tc_ptx.cuh"
#include "kvq_mma_ptx.cuh"
#include "kvq_prefill.cuh"
#include "kvq_prefill_body.cuh"

namespace kvq {
namespace {

using namespace ptx;

constexpr int PD = 128;              // head_dim
constexpr int PROWS = 128;           // (query, head) rows per CTA
constexpr int PTILE = 64;            // positions per tile (one page)
constexpr int PTHREADS = 256;        // 8 warps x 16 rows
constexpr unsigned kFull = 0xffffffffu;

// shared memory: keys hi/lo [64 pos][128 ch] bf16, values hi/lo [128 ch][64 pos]
// bf16, value (scale 2^vb, zero - scale 2^vb) [64][nvg] float pairs, and two
// stages of a page's raw blocks (key codes, key metadata, value codes, value
// metadata), the next tile's copied while the current one is worked on
constexpr int KBYTES = PTILE * PD * 2;    // 16 KB per array
constexpr int NVG_MAX = 8;                // value groups of 16 channels or more
__host__ __device__ constexpr int raw_bytes(int kb, int vb, int nvg) {
    return PTILE * PD * kb / 8 + PTILE * (PD / 32) * 4 + PD * PTILE * vb / 8 + PTILE * nvg * 4;
}
constexpr int QFRAG_BYTES = 8 * 2 * 32 * 16;   // per warp: the query's A fragments [k-step][hi/lo][lane]
constexpr size_t prefill_mma_smem(int kb, int vb, int nvg) {
    return 4 * size_t(KBYTES) + size_t(PTILE) * nvg * 8 + 2 * size_t(raw_bytes(kb, vb, nvg)) +
           size_t(PTHREADS / 32) * QFRAG_BYTES;
}

// the N words of bytes [4 N k, 4 N (k + 1)) of row r of a chunk-major block
// [chunk][rows][cw] of ROWB-byte rows (cw = min(16, ROWB)), as vector loads
template <int N, int ROWB>
__device__ __forceinline__ void row_words(const uint8_t* blk, int rows, int r, int k, uint32_t (&w)[N]) {
    constexpr int cw = ROWB < 16 ? ROWB : 16;
    static_assert(4 * N <= cw || 4 * N % cw == 0, "a word group is inside one chunk or whole chunks");
    const int byte = 4 * N * k;
    const uint8_t* a = blk + (byte / cw) * (rows * cw) + r * cw + (byte % cw);
    if constexpr (N == 1) {
        w[0] = *reinterpret_cast<const uint32_t*>(a);
    } else if constexpr (N == 2) {
        const uint2 u = *reinterpret_cast<const uint2*>(a);
        w[0] = u.x, w[1] = u.y;
    } else if constexpr (N == 4) {
        const uint4 u = *reinterpret_cast<const uint4*>(a);
        w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
    } else {
        const uint4 u = *reinterpret_cast<const uint4*>(a);
        const uint4 u2 = *reinterpret_cast<const uint4*>(a + rows * cw);
        w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w, w[4] = u2.x, w[5] = u2.y, w[6] = u2.z, w[7] = u2.w;
    }
}

__device__ __forceinline__ void cpa16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ float bits_bf16(uint32_t b) { return __uint_as_float(b << 16); }
__device__ __forceinline__ float bits_half(uint32_t b) {
    __half_raw r;
    r.x = uint16_t(b);
    return __half2float(__half(r));
}
// two values (first in the low half) as packed bf16 hi and lo words:
// hi = bf16(x), lo = bf16(x - hi), two values per conversion
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xffff0000u));
    lo = *reinterpret_cast<const uint32_t*>(&l);
}
// code c (BITS wide) at bit sh of x as the float 1 + c 2^-BITS (the code in the
// top of the mantissa of 1.0f): scale*c + zero = (scale 2^BITS) f + (zero - scale 2^BITS)
template <int BITS>
__device__ __forceinline__ float code_f(uint32_t x, int sh) {
    constexpr int top = 23 - BITS;
    constexpr uint32_t mask = ((1u << BITS) - 1u) << top;
    const uint32_t y = sh <= top ? (x << (top - sh)) : (x >> (sh - top));
    return __uint_as_float((y & mask) | 0x3F800000u);
}
// byte offset of 16-byte chunk c of row r in a [rows][chunks_per_row] array swizzled by row
__device__ __forceinline__ uint32_t swz(int r, int c, int chunks_per_row) {
    return uint32_t(r * chunks_per_row + (c ^ (r & 7))) * 16u;
}

template <int KB, int VB>
__global__ void __launch_bounds__(PTHREADS, 1) prefill_mma_kernel(const prefill::View v) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sKh = smem_u32(smem), sKl = sKh + KBYTES, sVh = sKl + KBYTES, sVl = sVh + KBYTES;
    float2* sVf = reinterpret_cast<float2*>(smem + 4 * KBYTES);       // [64][nvg]
    // raw page blocks of a tile: [stage][key codes | key metadata | value codes | value metadata]
    const int KCB = PTILE * PD * KB / 8, KMB = PTILE * (PD / 32) * 4, VCB = PD * PTILE * VB / 8;
    const int RAWB = raw_bytes(KB, VB, v.nvg);
    uint8_t* raw0 = smem + 4 * KBYTES + size_t(PTILE) * v.nvg * 8;
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g8 = lane >> 2, tig = lane & 3;
    const int g = v.g, QT = PROWS / g, R = QT * g;
    const int L = min(v.lens[b], v.len_cap);
    const int q0 = v.cu_q[b], n = v.cu_q[b + 1] - q0;
    if (n <= 0 || n > L || n > v.max_q) return;            // uniform over the CTA
    const int i0 = qt * QT;
    if (i0 >= n) return;
    const int nq = min(QT, n - i0);
    const int base = L - n;                                // position of query 0 of the chunk
    const int p_max = base + i0 + nq - 1;
    const int Lq = L - v.W > 0 ? L - v.W : 0;              // positions below Lq live in pages

    // ---- this warp's rows as A fragments (query pre-scaled to the log2 domain)
    const int r_lo = 16 * warp + g8, r_hi = r_lo + 8;     // the lane's two rows
    auto row_valid = [&](int r) { return r < R && r / g < nq; };
    auto row_pos = [&](int r) { return row_valid(r) ? base + i0 + r / g : -1; };
    const int p_lo = row_pos(r_lo), p_hi = row_pos(r_hi);
    // the query's A fragments (bf16 hi and lo parts) in shared memory, each lane's
    // own in register order, read back per k-step (registers for the tiles' work)
    uint4* sQ = reinterpret_cast<uint4*>(raw0 + 2 * size_t(RAWB)) + size_t(warp) * (QFRAG_BYTES / 16);
    {
        auto qpair = [&](int r, int ch, uint32_t& hi, uint32_t& lo) {
            float x0 = 0.0f, x1 = 0.0f;
            if (row_valid(r)) {
                const size_t idx = (size_t(q0 + i0 + r / g) * v.hq + size_t(h) * g + r % g) * PD + ch;
                if (v.q_bf16) {
                    const uint32_t w2 = *reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(v.q) + idx);
                    x0 = bits_bf16(w2 & 0xffffu);
                    x1 = bits_bf16(w2 >> 16);
                } else {
                    const float2 f = *reinterpret_cast<const float2*>(static_cast<const float*>(v.q) + idx);
                    x0 = f.x;
                    x1 = f.y;
                }
            }
            split2(x0 * v.scale_log2, x1 * v.scale_log2, hi, lo);
        };
#pragma unroll 2
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t hq[4], lq[4];
            qpair(r_lo, 16 * kk + 2 * tig, hq[0], lq[0]);
            qpair(r_hi, 16 * kk + 2 * tig, hq[1], lq[1]);
            qpair(r_lo, 16 * kk + 8 + 2 * tig, hq[2], lq[2]);
            qpair(r_hi, 16 * kk + 8 + 2 * tig, hq[3], lq[3]);
            sQ[(2 * kk) * 32 + lane] = make_uint4(hq[0], hq[1], hq[2], hq[3]);
            sQ[(2 * kk + 1) * 32 + lane] = make_uint4(lq[0], lq[1], lq[2], lq[3]);
        }
    }
    float o[16][4];
#pragma unroll
    for (int c = 0; c < 16; ++c) o[c][0] = o[c][1] = o[c][2] = o[c][3] = 0.0f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.0f, l_hi = 0.0f;   // per-lane partial sums
    const int warp_pmax = max(p_lo, p_hi);                 // newest position this lane's rows see

    const size_t blk = size_t(h);                          // kv-head index inside a page block
    // page of tile index lp (-1: unmapped, or not a paged tile)
    auto page_of = [&](int lp) -> int {
        if (lp * PTILE >= Lq || lp * PTILE > p_max || lp >= v.max_pages) return -1;
        const int pg = v.page_table[size_t(b) * v.max_pages + lp];
        return pg >= v.num_pages ? -1 : pg;
    };
    // this thread's 16-byte pieces of the raw blocks of page pg into stage st
    auto issue = [&](int pg, int st) {
        if (pg < 0) return;
        const uint32_t d0 = smem_u32(raw0 + size_t(st) * RAWB);
        const size_t bk = size_t(pg) * v.hkv + blk;
        const uint8_t* kc = v.k_codes + bk * size_t(KCB);
        const uint8_t* km = reinterpret_cast<const uint8_t*>(v.k_meta) + bk * size_t(KMB);
        const uint8_t* vc = v.v_codes + bk * size_t(VCB);
        const uint8_t* vm = reinterpret_cast<const uint8_t*>(v.v_meta) + bk * size_t(PTILE * v.nvg * 4);
        for (int c = tid; c < KCB / 16; c += PTHREADS) cpa16(d0 + 16 * c, kc + 16 * c);
        for (int c = tid; c < KMB / 16; c += PTHREADS) cpa16(d0 + KCB + 16 * c, km + 16 * c);
        for (int c = tid; c < VCB / 16; c += PTHREADS) cpa16(d0 + KCB + KMB + 16 * c, vc + 16 * c);
        for (int c = tid; c < PTILE * v.nvg * 4 / 16; c += PTHREADS) cpa16(d0 + KCB + KMB + VCB + 16 * c, vm + 16 * c);
    };
    int pg = page_of(0), pg_next = page_of(1), pg_after = page_of(2);
    issue(pg, 0);
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int t0 = 0, st = 0; t0 <= p_max; t0 += PTILE, st ^= 1) {
        // the next tile's copies go to the other stage, free since the last
        // tile's reconstruction (before the barrier that preceded its products)
        issue(pg_next, st ^ 1);
        asm volatile("cp.async.commit_group;" ::: "memory");
        const int pg_later = page_of(t0 / PTILE + 3);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncthreads();                                   // this tile's pieces have landed; the previous tile's readers are done
        const uint8_t* raw = raw0 + size_t(st) * RAWB;
        // value metadata of the tile's paged positions, as (scale 2^VB, zero - scale 2^VB)
        if (pg >= 0)
            for (int e = tid; e < PTILE * v.nvg; e += PTHREADS) {
                const uint32_t m = reinterpret_cast<const uint32_t*>(raw + KCB + KMB + VCB)[e];
                const float sc = bits_half(m & 0xffffu) * float(1 << VB);
                sVf[e] = make_float2(sc, bits_half(m >> 16) - sc);
            }
        __syncthreads();
        // ---- keys: thread = (position, key group of 32 channels), 8 channels at a time
        {
            // a warp: 32 consecutive positions of one key group (conflict-free row reads)
            const int t = tid & (PTILE - 1), grp = tid / PTILE, pos = t0 + t;
            // 0: zeros (past every row, or an unmapped page), 1: page codes, 2: window row
            const int kind = pos > p_max ? 0 : (pos < Lq ? (pg >= 0 ? 1 : 0) : 2);
            uint32_t wd[KB];
            float sc = 0.0f, zr = 0.0f;
            const uint16_t* wrow = nullptr;
            if (kind == 1) {
                row_words<KB, PD * KB / 8>(raw, PTILE, t, grp, wd);      // 32 channels of KB bits: KB words
                const uint32_t m = reinterpret_cast<const uint32_t*>(raw + KCB)[t * (PD / 32) + grp];
                sc = bits_half(m & 0xffffu) * float(1 << KB);
                zr = bits_half(m >> 16) - sc;
            } else if (kind == 2) {
                wrow = v.k_win + ((size_t(b) * v.hkv + blk) * v.W + size_t(pos % v.W)) * PD + 32 * grp;
            }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t hi[4], lo[4];
                if (kind == 2) {
                    const uint4 u = reinterpret_cast<const uint4*>(wrow)[cc];   // bf16 rows: lo parts are zero
                    hi[0] = u.x, hi[1] = u.y, hi[2] = u.z, hi[3] = u.w;
                    lo[0] = lo[1] = lo[2] = lo[3] = 0u;
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float x2[2] = {0.0f, 0.0f};
                        if (kind == 1) {
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int j = 8 * cc + 2 * k + e;
                                x2[e] = fmaf(code_f<KB>(wd[(j * KB) >> 5], (j * KB) & 31), sc, zr);
                            }
                        }
                        split2(x2[0], x2[1], hi[k], lo[k]);
                    }
                }
                const uint32_t off = swz(t, 4 * grp + cc, 16);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(sKh + off), "r"(hi[0]), "r"(hi[1]),
                             "r"(hi[2]), "r"(hi[3])
                             : "memory");
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(sKl + off), "r"(lo[0]), "r"(lo[1]),
                             "r"(lo[2]), "r"(lo[3])
                             : "memory");
            }
        }
        // ---- values: thread = (channel, half of the tile's positions), 8 positions at a time
        {
            const int ch = tid >> 1, half = tid & 1, gvc = ch / v.vg;
            uint32_t wd[VB];
            if (pg >= 0) {
                row_words<VB, PTILE * VB / 8>(raw + KCB + KMB, PD, ch, half, wd);   // 32 positions: VB words
            }
            const uint16_t* vw = reinterpret_cast<const uint16_t*>(v.v_win);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float x2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int i = 8 * cc + 2 * k + e, t = 32 * half + i, pos = t0 + t;
                        float xv = 0.0f;
                        if (pos <= p_max) {
                            if (pos < Lq) {
                                if (pg >= 0) {
                                    const float2 sz = sVf[t * v.nvg + gvc];
                                    xv = fmaf(code_f<VB>(wd[(i * VB) >> 5], (i * VB) & 31), sz.x, sz.y);
                                }
                            } else {
                                xv = bits_bf16(vw[((size_t(b) * v.hkv + blk) * v.W + size_t(pos % v.W)) * PD + ch]);
                            }
                        }
                        x2[e] = xv;
                    }
                    split2(x2[0], x2[1], hi[k], lo[k]);
                }
                const uint32_t off = swz(ch, 4 * half + cc, 8);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(sVh + off), "r"(hi[0]), "r"(hi[1]),
                             "r"(hi[2]), "r"(hi[3])
                             : "memory");
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(sVl + off), "r"(lo[0]), "r"(lo[1]),
                             "r"(lo[2]), "r"(lo[3])
                             : "memory");
            }
        }
        __syncthreads();
        pg = pg_next;
        pg_next = pg_after;
        pg_after = pg_later;
        // no row of this warp sees the tile (every lane takes the vote)
        const bool skip = __all_sync(kFull, warp_pmax < t0);
        if (skip) continue;

        // ---- scores of the warp's 16 rows x 64 positions
        // (k-step outer: eight independent accumulators between dependent MMAs)
        float s[8][4];
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint4 a = sQ[(2 * kk) * 32 + lane], c = sQ[(2 * kk + 1) * 32 + lane];
            const uint32_t qh[4] = {a.x, a.y, a.z, a.w}, ql[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t f[4];      // Kh k0-7, Kh k8-15, Kl k0-7, Kl k8-15 of positions 8j .. 8j+7
                ldsm_x4(f, (mi < 2 ? sKh : sKl) + swz(8 * j + rr, 2 * kk + (mi & 1), 16));
                mma_bf16(s[j], qh, f[0], f[1]);
                mma_bf16(s[j], qh, f[2], f[3]);
                mma_bf16(s[j], ql, f[0], f[1]);
            }
        }
        // ---- causal mask, online softmax (rows r_lo: s[][0..1], r_hi: s[][2..3])
        float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int pos = t0 + 8 * j + 2 * tig;
            if (pos > p_lo) s[j][0] = -INFINITY;
            if (pos + 1 > p_lo) s[j][1] = -INFINITY;
            if (pos > p_hi) s[j][2] = -INFINITY;
            if (pos + 1 > p_hi) s[j][3] = -INFINITY;
            mx_lo = fmaxf(mx_lo, fmaxf(s[j][0], s[j][1]));
            mx_hi = fmaxf(mx_hi, fmaxf(s[j][2], s[j][3]));
        }
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(kFull, mx_lo, 1));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(kFull, mx_lo, 2));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(kFull, mx_hi, 1));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(kFull, mx_hi, 2));
        const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
        const float mu_lo = mn_lo == -INFINITY ? 0.0f : mn_lo, mu_hi = mn_hi == -INFINITY ? 0.0f : mn_hi;
        const float a_lo = exp2f(m_lo - mu_lo), a_hi = exp2f(m_hi - mu_hi);   // 0 while m was -inf
        m_lo = mn_lo;
        m_hi = mn_hi;
        float ps_lo = 0.0f, ps_hi = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            s[j][0] = exp2f(s[j][0] - mu_lo);
            s[j][1] = exp2f(s[j][1] - mu_lo);
            s[j][2] = exp2f(s[j][2] - mu_hi);
            s[j][3] = exp2f(s[j][3] - mu_hi);
            ps_lo += s[j][0] + s[j][1];
            ps_hi += s[j][2] + s[j][3];
        }
        l_lo = fmaf(l_lo, a_lo, ps_lo);
        l_hi = fmaf(l_hi, a_hi, ps_hi);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            o[c][0] *= a_lo;
            o[c][1] *= a_lo;
            o[c][2] *= a_hi;
            o[c][3] *= a_hi;
        }
        // ---- O += P V: P's A fragments from the score registers, 16 positions per step
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t ph[4], pl[4];
            split2(s[2 * kk][0], s[2 * kk][1], ph[0], pl[0]);
            split2(s[2 * kk][2], s[2 * kk][3], ph[1], pl[1]);
            split2(s[2 * kk + 1][0], s[2 * kk + 1][1], ph[2], pl[2]);
            split2(s[2 * kk + 1][2], s[2 * kk + 1][3], ph[3], pl[3]);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                uint32_t f[4];      // Vh k0-7, Vh k8-15, Vl k0-7, Vl k8-15 of channels 8c .. 8c+7
                ldsm_x4(f, (mi < 2 ? sVh : sVl) + swz(8 * c + rr, 2 * kk + (mi & 1), 8));
                mma_bf16(o[c], ph, f[0], f[1]);
                mma_bf16(o[c], ph, f[2], f[3]);
                mma_bf16(o[c], pl, f[0], f[1]);
            }
        }
    }

    asm volatile("cp.async.wait_group 0;" ::: "memory");   // nothing in flight when the CTA exits

    // ---- o / l and lse = (m + log2 l) ln 2
    l_lo += __shfl_xor_sync(kFull, l_lo, 1);
    l_lo += __shfl_xor_sync(kFull, l_lo, 2);
    l_hi += __shfl_xor_sync(kFull, l_hi, 1);
    l_hi += __shfl_xor_sync(kFull, l_hi, 2);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int r = half ? r_hi : r_lo;
        if (!row_valid(r)) continue;
        const float l = half ? l_hi : l_lo, m = half ? m_hi : m_lo;
        const size_t orow = size_t(q0 + i0 + r / g) * v.hq + size_t(h) * g + r % g;
        const float inv = 1.0f / l;
        float* dst = v.out + orow * PD;
#pragma unroll
        for (int c = 0; c < 16; ++c)
            *reinterpret_cast<float2*>(dst + 8 * c + 2 * tig) =
                make_float2(o[c][2 * half] * inv, o[c][2 * half + 1] * inv);
        if (v.lse && tig == 0) v.lse[orow] = (m + log2f(l)) * 0.693147180559945309f;
    }
}

template <int KB, int VB>
cudaError_t launch_kv(const prefill::View& v, cudaStream_t s) {
    static bool configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(prefill_mma_kernel<KB, VB>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   int(prefill_mma_smem(KB, VB, NVG_MAX)));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const int qpc = PROWS / v.g;
    dim3 grid((v.max_q + qpc - 1) / qpc, v.hkv, v.batch);
    prefill_mma_kernel<KB, VB><<<grid, PTHREADS, prefill_mma_smem(KB, VB, v.nvg), s>>>(v);
    return cudaGetLastError();
}

template <int KB>
cudaError_t launch_k(const prefill::View& v, cudaStream_t s) {
    switch (v.vb) {
        case 1: return launch_kv<KB, 1>(v, s);
        case 2: return launch_kv<KB, 2>(v, s);
        case 4: return launch_kv<KB, 4>(v, s);
        default: return launch_kv<KB, 8>(v, s);
    }
}

}  // namespace

bool prefill_mma_supported(const prefill::View& v) {
    return v.d == PD && !v.kpc && !v.rotate && !v.one_query && v.kg == 32 && v.g >= 1 && v.g <= 8 &&
           PD % v.vg == 0 && v.vg >= 16 && (v.kb == 1 || v.kb == 2 || v.kb == 4 || v.kb == 8) &&
           (v.vb == 1 || v.vb == 2 || v.vb == 4 || v.vb == 8);
}

cudaError_t launch_prefill_mma(const prefill::View& v, cudaStream_t s) {
    switch (v.kb) {
        case 1: return launch_k<1>(v, s);
        case 2: return launch_k<2>(v, s);
        case 4: return launch_k<4>(v, s);
        default: return launch_k<8>(v, s);
    }
}

}  // namespace kvq

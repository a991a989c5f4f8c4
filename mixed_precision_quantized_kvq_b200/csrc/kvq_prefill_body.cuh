// Chunked-prefill attention over the quantized cache: the work of one CTA.
//
// A chunk of n new tokens of a sequence has been appended, so the sequence
// holds L positions and its queries sit at positions L-n .. L-1.  Query i
// attends, causally, to positions [0, L-n+i] as the cache holds them: pages
// (group-quantized codes, reconstructed as code*scale + zero in fp32) below
// L-W, the bf16 window from there on ("Kuantisasi KV cache mengganggu
// attention ...", sections "Error pada key masuk sebelum softmax" for
// s = qK^T/sqrt(d), a = softmax(s), o = aV, and "Pertumbuhan cache mengubah
// trade pada serving" for the recent tokens kept in higher precision and for
// dequantization fused into attention).  With key rotation, page keys are in
// the rotated domain and are scored with the rotated query; window keys with
// the plain one ("Quantize What Counts ...", Resultaten: rotation on keys).
//
// One CTA takes 64 (query, head) rows of one (sequence, kv-head): the
// 64/g newest-to-be queries of a query tile, each with the g query heads of
// the kv-group.  It walks the positions in 64-position tiles (one page),
// stages the tile's keys and values into shared memory as fp32, forms the
// 64x64 score block, updates a running max and sum per row (flash-style
// online softmax in the log2 domain) and accumulates the output in
// registers.  CUDA cores only.
//
// The body is written against a small context object (thread and block
// indices, block barrier, warp max and sum, shared memory) so that the same
// code runs as the CUDA kernel and, for tests, as host C++ with one thread
// per CUDA thread.  Nothing here is CUDA-only beyond what the context
// provides.
#pragma once

#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#include <cuda_fp16.h>

#ifndef KVQ_HD
#define KVQ_HD __host__ __device__ __forceinline__
#endif

namespace kvq {
namespace prefill {

constexpr int kRows = 64;      // (query, head) rows per CTA
constexpr int kTile = 64;      // positions per tile: one page
constexpr int kThreads = 256;  // 8 warps

// Everything one launch reads: the cache view and the call's arguments.
struct View {
    int d, hq, hkv, g;
    int kb, vb, kg, vg, nkg, nvg;
    int W, rotate;
    int kpc;                           // 1: key groups of kg positions of one channel
    int R;                             // ring slots: W, or W + kg - 1 with kpc
    const int8_t* signs;               // [d] +-1, when rotating
    const uint8_t* k_codes;
    const uint8_t* v_codes;
    const uint32_t* k_meta;            // {u16 scale, u16 zero} per group
    const uint32_t* v_meta;
    const uint16_t* k_win;             // bf16 bit patterns [B][Hkv][W][d]
    const uint16_t* v_win;
    const int32_t* page_table;         // [B][max_pages]
    int batch, max_pages, num_pages;
    int krow_bytes, vchan_bytes, kch, vch;
    int kchan_bytes, kchc;             // kpc: key channel run bytes and chunk bytes
    const void* q;                     // [total_q][Hq][d], bf16 or fp32
    int q_bf16;
    int one_query;                     // decode: one query per sequence, q row b, cu_q unused;
                                       // an empty sequence gets out = 0, lse = -inf
    const int32_t* cu_q;               // [B+1] query row offsets
    const int32_t* lens;               // [B] positions, the chunk included
    int len_cap;                       // lengths above it are clamped to it
    int max_q;                         // >= every chunk length
    float scale_log2;                  // softmax scale * log2(e)
    float* out;                        // [total_q][Hq][d]
    float* lse;                        // [total_q][Hq] natural log, or null
};

KVQ_HD int imin(int a, int b) { return a < b ? a : b; }

// queries per CTA for a kv-group of g query heads
KVQ_HD int queries_per_cta(int g) { return kRows / g; }

// shared memory of one CTA (bytes)
KVQ_HD size_t smem_bytes(int d, int rotate) {
    const size_t ld = size_t(d) + 4;
    const size_t floats = size_t(kRows) * ld * (rotate ? 2 : 1)   // queries (and rotated queries)
                          + 2 * size_t(kTile) * ld                 // keys, values of a tile
                          + size_t(kRows) * (kTile + 4)            // scores / weights
                          + 3 * size_t(kRows);                     // running max, sum, rescale
    return floats * 4 + size_t(kTile) * 4;                        // + page flag per position
}

KVQ_HD float bf16_bits_f32(uint16_t b) {
    const uint32_t u = uint32_t(b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

KVQ_HD float half_bits_f32(uint16_t b) {
    __half_raw r;
    r.x = b;
    return __half2float(__half(r));
}

// positions of a length-L sequence that live in pages: below L - W, rounded
// down to whole key groups when key groups run along positions
KVQ_HD int paged_len(const View& v, int L) {
    const int q = L - v.W > 0 ? L - v.W : 0;
    return v.kpc ? q - q % v.kg : q;
}

// key of channel j at token slot t of page pg (fp32 reconstruction)
KVQ_HD float key_at(const View& v, int pg, int h, int t, int j) {
    if (v.kpc) {   // channel runs, metadata [64/kg][d]
        const int bit = t * v.kb, byte = bit >> 3;
        const uint8_t* blk = v.k_codes + (size_t(pg) * v.hkv + h) * size_t(v.d) * v.kchan_bytes;
        const uint8_t c8 = blk[(byte / v.kchc) * (v.d * v.kchc) + j * v.kchc + (byte % v.kchc)];
        const uint32_t code = (uint32_t(c8) >> (bit & 7)) & ((1u << v.kb) - 1u);
        const uint32_t m = v.k_meta[((size_t(pg) * v.hkv + h) * size_t(kTile / v.kg) + t / v.kg) * v.d + j];
        return fmaf(float(code), half_bits_f32(uint16_t(m & 0xffffu)), half_bits_f32(uint16_t(m >> 16)));
    }
    const int bit = j * v.kb, byte = bit >> 3;
    const uint8_t* blk = v.k_codes + (size_t(pg) * v.hkv + h) * size_t(kTile) * v.krow_bytes;
    const uint8_t c8 = blk[(byte / v.kch) * (kTile * v.kch) + t * v.kch + (byte % v.kch)];
    const uint32_t code = (uint32_t(c8) >> (bit & 7)) & ((1u << v.kb) - 1u);
    const uint32_t m = v.k_meta[((size_t(pg) * v.hkv + h) * kTile + t) * v.nkg + j / v.kg];
    return fmaf(float(code), half_bits_f32(uint16_t(m & 0xffffu)), half_bits_f32(uint16_t(m >> 16)));
}

// value of channel j at token slot t of page pg (fp32 reconstruction)
KVQ_HD float value_at(const View& v, int pg, int h, int t, int j) {
    const int bit = t * v.vb, byte = bit >> 3;
    const uint8_t* blk = v.v_codes + (size_t(pg) * v.hkv + h) * size_t(v.d) * v.vchan_bytes;
    const uint8_t c8 = blk[(byte / v.vch) * (v.d * v.vch) + j * v.vch + (byte % v.vch)];
    const uint32_t code = (uint32_t(c8) >> (bit & 7)) & ((1u << v.vb) - 1u);
    const uint32_t m = v.v_meta[((size_t(pg) * v.hkv + h) * kTile + t) * v.nvg + j / v.vg];
    return fmaf(float(code), half_bits_f32(uint16_t(m & 0xffffu)), half_bits_f32(uint16_t(m >> 16)));
}

#ifdef __CUDACC__
#pragma nv_exec_check_disable
#endif
template <int D, class Ctx>
KVQ_HD void body(Ctx& cx, const View& v) {
    constexpr int LD = D + 4;        // padded row of queries, keys, values
    constexpr int LP = kTile + 4;    // padded row of scores
    constexpr int CPT = D / 16;      // output columns per thread
    const int qt = cx.bx(), h = cx.by(), b = cx.bz();
    const int tid = cx.tid();
    const int g = v.g, QT = kRows / g, R = QT * g;
    const int L = imin(v.lens[b], v.len_cap);
    if (v.one_query && L <= 0) {                           // empty sequence: o = 0, lse = -inf
        if (qt == 0)
            for (int e = tid; e < g * D; e += kThreads) {
                const size_t orow = size_t(b) * v.hq + size_t(h) * g + e / D;
                v.out[orow * D + e % D] = 0.f;
                if (v.lse && e % D == 0) v.lse[orow] = -INFINITY;
            }
        return;
    }
    const int q0 = v.one_query ? b : v.cu_q[b];
    const int n = v.one_query ? 1 : v.cu_q[b + 1] - q0;
    if (n <= 0 || n > L || n > v.max_q) return;           // uniform over the CTA
    const int i0 = qt * QT;
    if (i0 >= n) return;
    const int nq = imin(QT, n - i0);                       // queries of this CTA
    const int base = L - n;                                // position of query 0 of the chunk
    const int p_max = base + i0 + nq - 1;                  // newest position any row sees
    const int Lq = paged_len(v, L);                        // positions below Lq live in pages

    float* sQ = cx.smem();
    float* sQr = sQ + kRows * LD;
    float* sK = sQ + kRows * LD * (v.rotate ? 2 : 1);
    float* sV = sK + kTile * LD;
    float* sP = sV + kTile * LD;
    float* sM = sP + kRows * LP;
    float* sL = sM + kRows;
    float* sA = sL + kRows;
    int* sPaged = reinterpret_cast<int*>(sA + kRows);

    // ---- queries: row r = (query r/g of the tile, head r%g of the group) ----
    for (int e = tid; e < kRows * D; e += kThreads) {
        const int r = e / D, j = e % D, qi = r / g, hr = r % g;
        float x = 0.f;
        if (r < R && qi < nq) {
            const size_t idx = (size_t(q0 + i0 + qi) * v.hq + size_t(h) * g + hr) * D + j;
            x = v.q_bf16 ? bf16_bits_f32(static_cast<const uint16_t*>(v.q)[idx])
                         : static_cast<const float*>(v.q)[idx];
        }
        sQ[r * LD + j] = x;
        if (v.rotate) sQr[r * LD + j] = x * float(v.signs[j]);
    }
    if (tid < kRows) {
        sM[tid] = -INFINITY;
        sL[tid] = 0.f;
    }
    cx.sync();
    if (v.rotate) {
        // Sylvester-ordered Walsh-Hadamard transform of sign-flipped rows:
        // butterflies (a, b) -> (a + b, a - b) at strides 1 .. D/2, then 1/sqrt(D)
        for (int s = 1; s < D; s <<= 1) {
            for (int e = tid; e < kRows * (D / 2); e += kThreads) {
                const int r = e / (D / 2), k = e % (D / 2);
                const int j = (k / s) * 2 * s + (k % s);
                const float a = sQr[r * LD + j], c = sQr[r * LD + j + s];
                sQr[r * LD + j] = a + c;
                sQr[r * LD + j + s] = a - c;
            }
            cx.sync();
        }
        const float inv = D == 128 ? 0.0883883476483184405f : 0.125f;
        for (int e = tid; e < kRows * D; e += kThreads) sQr[(e / D) * LD + e % D] *= inv;
        cx.sync();
    }

    // score block: rows sr..sr+3, positions sc..sc+3; output block: rows pr..pr+3, columns pc..pc+CPT-1
    const int sr = (tid / 16) * 4, sc = (tid % 16) * 4;
    const int pr = (tid / 16) * 4, pc = (tid % 16) * CPT;
    int p_row[4];
    for (int i = 0; i < 4; ++i) {
        const int r = sr + i, qi = r / g;
        p_row[i] = (r < R && qi < nq) ? base + i0 + qi : p_max;   // padding rows: finite, unused
    }
    float o[4][CPT];
    for (int i = 0; i < 4; ++i)
        for (int c = 0; c < CPT; ++c) o[i][c] = 0.f;

    for (int t0 = 0; t0 <= p_max; t0 += kTile) {
        // ---- stage keys and values of positions t0 .. t0+63 (slot t of logical page t0/64) ----
        for (int e = tid; e < kTile * D; e += kThreads) {
            const int t = e / D, j = e % D, pos = t0 + t;
            float kx = 0.f, vx = 0.f;
            int paged = 0;
            if (pos <= p_max) {
                if (pos < Lq) {
                    paged = 1;
                    const int lp = pos / kTile;
                    const int pg = lp < v.max_pages ? v.page_table[size_t(b) * v.max_pages + lp] : -1;
                    if (pg >= 0 && pg < v.num_pages) {
                        kx = key_at(v, pg, h, t, j);
                        vx = value_at(v, pg, h, t, j);
                    }
                } else {
                    const size_t w = ((size_t(b) * v.hkv + h) * v.R + size_t(pos % v.R)) * D + j;
                    kx = bf16_bits_f32(v.k_win[w]);
                    vx = bf16_bits_f32(v.v_win[w]);
                }
            }
            sK[t * LD + j] = kx;
            sV[t * LD + j] = vx;
            if (j == 0) sPaged[t] = paged;
        }
        cx.sync();

        // ---- scores (log2 domain), causal mask ----
        {
            float acc[4][4];
            int paged[4];
            for (int c = 0; c < 4; ++c) paged[c] = sPaged[sc + c];
            for (int i = 0; i < 4; ++i)
                for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
            for (int k = 0; k < D; ++k) {
                float qa[4], qb[4], kk[4];
                for (int i = 0; i < 4; ++i) {
                    qa[i] = sQ[(sr + i) * LD + k];
                    qb[i] = v.rotate ? sQr[(sr + i) * LD + k] : qa[i];
                }
                for (int c = 0; c < 4; ++c) kk[c] = sK[(sc + c) * LD + k];
                for (int i = 0; i < 4; ++i)
                    for (int c = 0; c < 4; ++c) acc[i][c] = fmaf(paged[c] ? qb[i] : qa[i], kk[c], acc[i][c]);
            }
            for (int i = 0; i < 4; ++i)
                for (int c = 0; c < 4; ++c) {
                    const int pos = t0 + sc + c;
                    sP[(sr + i) * LP + sc + c] = pos <= p_row[i] ? acc[i][c] * v.scale_log2 : -INFINITY;
                }
        }
        cx.sync();

        // ---- online softmax: one warp per 8 rows, two positions per lane ----
        {
            const int warp = tid / 32, lane = tid % 32;
            for (int rr = 0; rr < kRows / (kThreads / 32); ++rr) {
                const int r = warp * (kRows / (kThreads / 32)) + rr;
                float* row = sP + r * LP;
                const float x0 = row[lane], x1 = row[lane + 32];
                const float mx = cx.warp_max(fmaxf(x0, x1));
                const float m_old = sM[r];
                const float m_new = fmaxf(m_old, mx);        // finite: position 0 is in every row's tile 0
                const float p0 = exp2f(x0 - m_new), p1 = exp2f(x1 - m_new);
                const float sum = cx.warp_sum(p0 + p1);
                const float alpha = exp2f(m_old - m_new);
                row[lane] = p0;
                row[lane + 32] = p1;
                if (lane == 0) {
                    sL[r] = sL[r] * alpha + sum;
                    sM[r] = m_new;
                    sA[r] = alpha;
                }
            }
        }
        cx.sync();

        // ---- o = o * alpha + P V ----
        for (int i = 0; i < 4; ++i) {
            const float a = sA[pr + i];
            for (int c = 0; c < CPT; ++c) o[i][c] *= a;
        }
        for (int t = 0; t < kTile; ++t) {
            float pp[4], vv[CPT];
            for (int i = 0; i < 4; ++i) pp[i] = sP[(pr + i) * LP + t];
            for (int c = 0; c < CPT; ++c) vv[c] = sV[t * LD + pc + c];
            for (int i = 0; i < 4; ++i)
                for (int c = 0; c < CPT; ++c) o[i][c] = fmaf(pp[i], vv[c], o[i][c]);
        }
        cx.sync();
    }

    // ---- o / l, lse = (m + log2 l) * ln 2 ----
    for (int i = 0; i < 4; ++i) {
        const int r = pr + i, qi = r / g, hr = r % g;
        if (r >= R || qi >= nq) continue;
        const size_t orow = size_t(q0 + i0 + qi) * v.hq + size_t(h) * g + hr;
        const float l = sL[r];
        float* dst = v.out + orow * D + pc;
        for (int c = 0; c < CPT; ++c) dst[c] = o[i][c] / l;
        if (v.lse && (tid % 16) == 0) v.lse[orow] = (sM[r] + log2f(l)) * 0.693147180559945309f;
    }
}

}  // namespace prefill
}  // namespace kvq

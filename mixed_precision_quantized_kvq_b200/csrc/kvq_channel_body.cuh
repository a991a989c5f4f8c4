// Per-channel key groups: the work of one CTA of the append, ring-write and
// dequantize kernels.
//
// "Kuantisasi KV cache mengganggu attention ...", section "Granularitas
// kuantisasi menentukan nilai yang berbagi scale": values that share a
// scale and zero point form a group, and the grouping axis may run along
// token positions.  Here a key group is kg consecutive positions of one
// channel, aligned to kg inside a 64-position page, with the same min/max
// quantizer as the per-token groups (fp16 zero rounded down, fp16 scale
// with every step rounded up, codes rint((x - zero) / scale) clamped).  A
// group is quantized once it is complete and out of the W newest positions
// (section "Pertumbuhan cache mengubah trade pada serving": recent tokens
// stay at higher precision), so positions below
// Q(L) = kg * floor(max(0, L - W) / kg) live in pages and the rest, W to
// W + kg - 1 of them, in a bf16 ring of R = W + kg - 1 slots.  Values keep
// per-token groups of vg channels.
//
// Storage of a (page, kv-head) block: key codes as channel runs of
// 64*kb/8 bytes (slot t in bits kb*(t mod 32/kb) of word t*kb/32),
// chunk-major in 16-byte chunks like the value runs; key metadata
// [64/kg][d] words {u16 scale, u16 zero}.
//
// The bodies take a context object (indices, barrier, shared memory, the
// IEEE operations with directed rounding, 32-bit atomics) so that the same
// code runs as CUDA kernels and, for tests, as host C++.
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
namespace chan {

constexpr int kPage = 64;
constexpr int kThreads = 128;

struct View {
    int d, hkv, kb, vb, kg, vg, nvg;
    int W, R;                          // window, ring slots (W + kg - 1)
    uint8_t* k_codes;
    uint8_t* v_codes;
    uint32_t* k_meta;                  // [pages][hkv][64/kg][d]
    uint32_t* v_meta;                  // [pages][hkv][64][d/vg]
    uint16_t* k_win;                   // bf16 bits [B][hkv][R][d]
    uint16_t* v_win;
    const int32_t* page_table;
    int batch, max_pages, num_pages;
    int kchan_bytes, vchan_bytes, kch, vch;   // run bytes, chunk bytes
    // append
    const void* k_new;
    const void* v_new;
    int in_bf16;
    const int32_t* cu_new;
    const int32_t* lens;               // append: before the new tokens; dequantize: lengths
    // dequantize
    float* k_out;
    float* v_out;
    int max_len;
};

KVQ_HD int imin(int a, int b) { return a < b ? a : b; }
KVQ_HD int imax(int a, int b) { return a > b ? a : b; }

// positions of a length-L sequence that live in pages
KVQ_HD int paged_len(int L, int W, int kg) {
    const int q = L - W > 0 ? L - W : 0;
    return q - q % kg;
}

KVQ_HD float bf16_f32(uint16_t b) {
    const uint32_t u = uint32_t(b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

KVQ_HD float half_f32(uint16_t b) {
    __half_raw r;
    r.x = b;
    return __half2float(__half(r));
}

KVQ_HD int phys_page(const View& v, int b, int lp) {
    if (lp < 0 || lp >= v.max_pages) return -1;
    const int pg = v.page_table[size_t(b) * v.max_pages + lp];
    return (pg >= 0 && pg < v.num_pages) ? pg : -1;
}

KVQ_HD uint8_t* k_block(const View& v, int pg, int h) {
    return v.k_codes + (size_t(pg) * v.hkv + h) * size_t(v.d) * v.kchan_bytes;
}
KVQ_HD uint8_t* v_block(const View& v, int pg, int h) {
    return v.v_codes + (size_t(pg) * v.hkv + h) * size_t(v.d) * v.vchan_bytes;
}
// byte `byte` of channel j's run in a block of chunk size ch
KVQ_HD size_t run_off(int d, int ch, int j, int byte) {
    return size_t(byte / ch) * (size_t(d) * ch) + size_t(j) * ch + size_t(byte % ch);
}
KVQ_HD uint32_t* k_meta_at(const View& v, int pg, int h, int slot, int j) {
    return v.k_meta + ((size_t(pg) * v.hkv + h) * size_t(kPage / v.kg) + slot / v.kg) * v.d + j;
}
KVQ_HD uint32_t* v_meta_at(const View& v, int pg, int h, int slot, int grp) {
    return v.v_meta + ((size_t(pg) * v.hkv + h) * kPage + slot) * v.nvg + grp;
}
KVQ_HD size_t ring_off(const View& v, int b, int h, int pos) {
    return ((size_t(b) * v.hkv + h) * v.R + size_t(pos % v.R)) * v.d;
}

// The quantizer of one group, in three parts so that several threads can
// share a group: the extremes of a part of the group, the metadata word
// {fp16 scale | fp16 zero << 16} of the group from its extremes (with the
// fp32 zero and scale the codes are formed with), and the codes of a part.
KVQ_HD void span_extremes(const float* x, int stride, int n, float& mn, float& mx) {
    mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        mn = fminf(mn, x[size_t(i) * stride]);
        mx = fmaxf(mx, x[size_t(i) * stride]);
    }
}
template <class Ctx>
KVQ_HD uint32_t span_meta(const Ctx& cx, float mn, float mx, int bits, float& zf, float& sf) {
    if (mn == 0.0f) mn = 0.0f;       // canonical +0
    if (mx == 0.0f) mx = 0.0f;
    const float qmax = float((1 << bits) - 1);
    const uint16_t zh = cx.f2h_rd(mn);
    zf = half_f32(zh);
    const float s32 = cx.div_ru(cx.sub_ru(mx, zf), qmax);
    uint16_t sh = cx.f2h_ru(s32);
    sf = half_f32(sh);
    if (sf == 0.0f) sh = 0;
    return uint32_t(sh) | (uint32_t(zh) << 16);
}
// codes of n values with the group's fp32 zero zf and scale sf:
// rint((x - zf) / sf) clamped to [0, 2^bits - 1], the quotient correctly
// rounded.  The quotient is formed as (x - zf) * (1 / sf), both correctly
// rounded, which is within 2^-22 |q| of the exact quotient; the two can round
// to different integers only when a half-integer lies that close to the
// product, and then the division is carried out (the codes are the same as
// with a division per value).
template <class Ctx>
KVQ_HD void span_codes(const Ctx& cx, const float* x, int stride, int n, float zf, float sf, float rs, int bits,
                       uint8_t* c) {
    const float qmax = float((1 << bits) - 1);
    for (int i = 0; i < n; ++i) {
        float code = 0.0f;
        if (sf != 0.0f) {
            const float a = cx.sub_rn(x[size_t(i) * stride], zf);
            float q = cx.mul_rn(a, rs);
            const float fq = floorf(q);
            if (fabsf(q - fq - 0.5f) <= fabsf(q) * 0x1p-20f) q = cx.div_rn(a, sf);
            code = fminf(fmaxf(rintf(q), 0.0f), qmax);
        }
        c[i] = uint8_t(code);
    }
}

// Write codes c[0], c[cs], ... of slots slot0 .. slot0+n-1 into channel j's
// run (bits per code `bits`).  Whole words are stored; words shared with
// another group (n*bits < 32) are merged bit-field by bit-field with
// atomics, since another CTA may write the rest of the word.
template <class Ctx>
KVQ_HD void put_run(const Ctx& cx, uint8_t* blk, int d, int ch, int j, int slot0, int n, int bits,
                    const uint8_t* c, int cs) {
    const int per_word = 32 / bits;
    const uint32_t cmask = (1u << bits) - 1u;
    const int w0 = slot0 / per_word, w1 = (slot0 + n + per_word - 1) / per_word;
    for (int w = w0; w < w1; ++w) {
        uint32_t val = 0, mask = 0;
        for (int i = 0; i < per_word; ++i) {
            const int t = w * per_word + i;
            if (t < slot0 || t >= slot0 + n) continue;
            mask |= cmask << (i * bits);
            val |= (uint32_t(c[size_t(t - slot0) * cs]) & cmask) << (i * bits);
        }
        uint32_t* at = reinterpret_cast<uint32_t*>(blk + run_off(d, ch, j, 4 * w));
        if (mask == 0xffffffffu) {
            *at = val;
        } else {
            cx.atomic_and(at, ~mask);
            cx.atomic_or(at, val);
        }
    }
}

// Threads of one append CTA on the GPU (the body works with any count).
constexpr int kGroupThreads = 512;
// Parts a group's values are split into between threads.
constexpr int kParts = 4;

// shared memory of one append CTA (bytes): keys and values as fp32 rows of
// d + 1 floats (the padding puts rows that different threads walk in
// different banks), the parts' extremes, per group (zero, scale, 1/scale),
// key codes [d][kg], value codes as rows of d + 4 bytes
KVQ_HD size_t append_smem_bytes(int d, int kg, int nvg) {
    return size_t(kg) * size_t(d + 1) * 8 + size_t(d + kg * nvg) * (kParts * 8 + 12) + size_t(d) * kg +
           size_t(kg) * size_t(d + 4);
}

struct alignas(16) Words4 {
    uint32_t w[4];
};

// Append, part 1.  CTA (gi, h, b): key group gi of the groups that this
// append completes for sequence b, kv-head h: its kg positions' keys and
// values (from the ring when older than L, else from the new rows) are
// quantized into their page.  Must run before part 2 rewrites ring slots.
// The CTA's groups (d key groups along positions, kg * nvg value groups
// along channels) are split into kParts parts each: the parts' extremes,
// then each group's metadata (one thread per group), then each part's codes,
// then the codes packed into the channel runs.
#ifdef __CUDACC__
#pragma nv_exec_check_disable
#endif
template <class Ctx>
KVQ_HD void append_groups_body(Ctx& cx, const View& v) {
    const int gi = cx.bx(), h = cx.by(), b = cx.bz(), tid = cx.tid(), NT = cx.nthreads();
    const int d = v.d, G = v.kg;
    const int L = v.lens[b], n = v.cu_new[b + 1] - v.cu_new[b];
    if (n <= 0 || L < 0) return;
    const int q0 = paged_len(L, v.W, G), q1 = paged_len(L + n, v.W, G);
    const int g0 = q0 + gi * G;
    if (g0 >= q1) return;
    const int pg = phys_page(v, b, g0 / kPage);
    if (pg < 0) return;
    const int slot0 = g0 % kPage;
    const int dp = d + 1, cp = d + 4;                         // padded row strides
    const int T = d + G * v.nvg;                              // groups: keys, then values
    float* sK = cx.smem();
    float* sV = sK + G * dp;
    float* sX = sV + G * dp;                                  // [T][kParts] {min, max}
    float* sQ = sX + 2 * T * kParts;                          // [T] {zero, scale, 1/scale}
    uint8_t* sKC = reinterpret_cast<uint8_t*>(sQ + 3 * T);    // key codes [d][G]
    uint8_t* sC = sKC + d * G;                                // value codes [G][d + 4]

    // positions still in the ring: 16-byte loads of 8 channels, every load of a
    // thread's batch issued before its stores (one memory latency per batch)
    const int nring = imax(0, imin(G, L - g0));
    const int d8 = d / 8, nvec = nring * d8;
    for (int base = 0; base < nvec; base += 8 * NT) {
        Words4 kk[8] = {}, vv[8] = {};
        for (int u = 0; u < 8; ++u) {
            const int e = base + u * NT + tid;
            if (e < nvec) {
                const size_t w = ring_off(v, b, h, g0 + e / d8) + 8 * size_t(e % d8);
                kk[u] = *reinterpret_cast<const Words4*>(v.k_win + w);
                vv[u] = *reinterpret_cast<const Words4*>(v.v_win + w);
            }
        }
        for (int u = 0; u < 8; ++u) {
            const int e = base + u * NT + tid;
            if (e >= nvec) continue;
            const int t = e / d8, j = 8 * (e % d8);
            for (int c = 0; c < 8; ++c) {
                sK[t * dp + j + c] = bf16_f32(uint16_t(kk[u].w[c >> 1] >> (16 * (c & 1))));
                sV[t * dp + j + c] = bf16_f32(uint16_t(vv[u].w[c >> 1] >> (16 * (c & 1))));
            }
        }
    }
    // positions among the new rows
    for (int e = nring * d + tid; e < G * d; e += NT) {
        const int t = e / d, j = e % d, pos = g0 + t;
        const size_t row = (size_t(v.cu_new[b] + pos - L) * v.hkv + h) * d + j;
        float kx, vx;
        if (v.in_bf16) {
            kx = bf16_f32(static_cast<const uint16_t*>(v.k_new)[row]);
            vx = bf16_f32(static_cast<const uint16_t*>(v.v_new)[row]);
        } else {
            kx = static_cast<const float*>(v.k_new)[row];
            vx = static_cast<const float*>(v.v_new)[row];
        }
        sK[t * dp + j] = kx;
        sV[t * dp + j] = vx;
    }
    cx.sync();
    // part e % kParts of group e / kParts: its values (x, stride, count)
    auto part = [&](int e, const float*& x, int& stride, int& m) {
        const int grp = e / kParts, k = e % kParts;
        if (grp < d) {                                        // key group: channel grp
            m = G / kParts;
            x = sK + size_t(k * m) * dp + grp;
            stride = dp;
        } else {                                              // value group: (position, channel group)
            const int t = (grp - d) / v.nvg, cg = (grp - d) % v.nvg;
            m = v.vg / kParts;
            x = sV + size_t(t) * dp + cg * v.vg + k * m;
            stride = 1;
        }
    };
    for (int e = tid; e < T * kParts; e += NT) {
        const float* x;
        int stride, m;
        part(e, x, stride, m);
        span_extremes(x, stride, m, sX[2 * e], sX[2 * e + 1]);
    }
    cx.sync();
    // each group's metadata once, from its parts' extremes
    for (int grp = tid; grp < T; grp += NT) {
        const float* ex = sX + 2 * grp * kParts;
        float mn = ex[0], mx = ex[1];
        for (int i = 1; i < kParts; ++i) {
            mn = fminf(mn, ex[2 * i]);
            mx = fmaxf(mx, ex[2 * i + 1]);
        }
        float zf, sf;
        const bool key = grp < d;
        const uint32_t meta = span_meta(cx, mn, mx, key ? v.kb : v.vb, zf, sf);
        if (key) {
            *k_meta_at(v, pg, h, slot0, grp) = meta;
        } else {
            const int t = (grp - d) / v.nvg, cg = (grp - d) % v.nvg;
            *v_meta_at(v, pg, h, slot0 + t, cg) = meta;
        }
        sQ[3 * grp] = zf;
        sQ[3 * grp + 1] = sf;
        sQ[3 * grp + 2] = sf != 0.0f ? cx.div_rn(1.0f, sf) : 0.0f;
    }
    cx.sync();
    for (int e = tid; e < T * kParts; e += NT) {
        const int grp = e / kParts, k = e % kParts;
        const float zf = sQ[3 * grp], sf = sQ[3 * grp + 1], rs = sQ[3 * grp + 2];
        const float* x;
        int stride, m;
        part(e, x, stride, m);
        if (grp < d) {
            span_codes(cx, x, stride, m, zf, sf, rs, v.kb, sKC + grp * G + k * m);
        } else {
            const int t = (grp - d) / v.nvg, cg = (grp - d) % v.nvg;
            span_codes(cx, x, stride, m, zf, sf, rs, v.vb, sC + t * cp + cg * v.vg + k * m);
        }
    }
    cx.sync();
    for (int e = tid; e < 2 * d; e += NT) {
        if (e < d) put_run(cx, k_block(v, pg, h), d, v.kch, e, slot0, G, v.kb, sKC + e * G, 1);
        else put_run(cx, v_block(v, pg, h), d, v.vch, e - d, slot0, G, v.vb, sC + (e - d), cp);
    }
}

// Append, part 2.  CTA (h, b): the new positions that stay in the window
// are written to their ring slots (fp32 input rounded to nearest-even bf16).
#ifdef __CUDACC__
#pragma nv_exec_check_disable
#endif
template <class Ctx>
KVQ_HD void ring_write_body(Ctx& cx, const View& v) {
    const int h = cx.bx(), b = cx.by(), tid = cx.tid();
    const int d = v.d;
    const int L = v.lens[b], n = v.cu_new[b + 1] - v.cu_new[b];
    if (n <= 0 || L < 0) return;
    const int w0 = imax(paged_len(L + n, v.W, v.kg), L);
    const int cnt = L + n - w0;
    for (int e = tid; e < cnt * d; e += cx.nthreads()) {
        const int pos = w0 + e / d, j = e % d;
        const size_t row = (size_t(v.cu_new[b] + pos - L) * v.hkv + h) * d + j;
        const size_t dst = ring_off(v, b, h, pos) + j;
        if (v.in_bf16) {
            v.k_win[dst] = static_cast<const uint16_t*>(v.k_new)[row];
            v.v_win[dst] = static_cast<const uint16_t*>(v.v_new)[row];
        } else {
            v.k_win[dst] = cx.f2bf_rn(static_cast<const float*>(v.k_new)[row]);
            v.v_win[dst] = cx.f2bf_rn(static_cast<const float*>(v.v_new)[row]);
        }
    }
}

// Dequantize (check path).  CTA (tile of 64 positions, h, b): positions
// below min(len, max_len) to fp32 [B][hkv][max_len][d]; page positions as
// code * scale + zero, ring positions as their bf16 values.
template <class Ctx>
KVQ_HD void dequant_body(Ctx& cx, const View& v) {
    const int tile = cx.bx(), h = cx.by(), b = cx.bz(), tid = cx.tid();
    const int d = v.d;
    const int L = v.lens[b];
    const int Lc = imin(L, v.max_len);
    const int Q = paged_len(L, v.W, v.kg);
    for (int e = tid; e < kPage * d; e += cx.nthreads()) {
        const int t = e / d, j = e % d, pos = tile * kPage + t;
        if (pos >= Lc) continue;
        const size_t o = ((size_t(b) * v.hkv + h) * v.max_len + pos) * d + j;
        if (pos >= Q) {
            const size_t w = ring_off(v, b, h, pos) + j;
            v.k_out[o] = bf16_f32(v.k_win[w]);
            v.v_out[o] = bf16_f32(v.v_win[w]);
            continue;
        }
        const int pg = phys_page(v, b, pos / kPage);
        if (pg < 0) continue;
        const int kbit = t * v.kb, vbit = t * v.vb;
        const uint32_t kc = (uint32_t(k_block(v, pg, h)[run_off(d, v.kch, j, kbit >> 3)]) >> (kbit & 7)) &
                            ((1u << v.kb) - 1u);
        const uint32_t vc = (uint32_t(v_block(v, pg, h)[run_off(d, v.vch, j, vbit >> 3)]) >> (vbit & 7)) &
                            ((1u << v.vb) - 1u);
        const uint32_t km = *k_meta_at(v, pg, h, t, j);
        const uint32_t vm = *v_meta_at(v, pg, h, t, j / v.vg);
        v.k_out[o] = fmaf(float(kc), half_f32(uint16_t(km & 0xffffu)), half_f32(uint16_t(km >> 16)));
        v.v_out[o] = fmaf(float(vc), half_f32(uint16_t(vm & 0xffffu)), half_f32(uint16_t(vm >> 16)));
    }
}

}  // namespace chan
}  // namespace kvq

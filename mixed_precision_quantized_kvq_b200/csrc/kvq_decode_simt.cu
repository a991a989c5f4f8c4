// Decode attention over the quantized cache on CUDA cores (all bit widths,
// head_dim 64/128, fp32 or bf16 query): split-K flash-decode with the
// dequantization fused into the score and value loops, and the log-sum-exp
// combine of the splits.
//
// Attention ("Kuantisasi KV cache mengganggu attention ...", section "Error
// pada key masuk sebelum softmax"): s = q K^T * sm_scale, a = softmax(s),
// o = a V.  Keys are never materialised: with x^ = c*scale + zero per group,
//   q . k^ = sum_groups ( scale * (q . c)_group + zero * (sum q)_group )
// and for values
//   o = sum_t p_t (scale_t c_t + zero_t) = sum_t (p_t scale_t) c_t + sum_t p_t zero_t.
// Section "Pertumbuhan cache mengubah trade pada serving": dequantization
// fused into the attention kernel; the newest W positions are read from the
// bf16 window.
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {

int g_decode_path = 0;

DecodePlan plan_decode(const Params& p, int batch, int max_len, int sm_count) {
    DecodePlan pl{};
    const int maxq = max_len - p.W > 0 ? max_len - p.W : 0;
    const int npages = (maxq + kPage - 1) / kPage;
    pl.window_split = p.W > 0 ? 1 : 0;
    const int units = batch * p.hkv > 0 ? batch * p.hkv : 1;
    if ((g_decode_path == 0 || g_decode_path == 2) && mma_supported(p, batch)) {
        // one CTA per SM at most, each with an equal share of the units; no
        // combine launch (split pairs are merged inside the kernel)
        const int win = p.W < max_len ? p.W : max_len;
        // an upper bound on the units (the kernel counts them from the device lengths)
        const long long nu = (long long)batch * p.hkv * ((maxq + 127) / 128 + (win + 15) / 16 + 1);
        pl.mma = 1;
        pl.ctas = (int)(nu < sm_count ? nu : sm_count);
        if (pl.ctas < 1) pl.ctas = 1;
        return pl;
    }
    pl.tc = (g_decode_path == 3 && tc_supported(p)) ? 1 : 0;
    if (pl.tc) {
        // quantized splits (slots 0 .. splits_q-1), each a whole number of
        // 128-token tiles, then the window CTAs (64 window positions each, short
        // enough to run in the slots the quantized splits leave free):
        // one wave of CTAs where the units allow it, at most 16 tiles per split
        const int win = p.W < max_len ? p.W : max_len;
        pl.window_split = win > 0 ? (win + kTcWindowPerCta - 1) / kTcWindowPerCta : 0;
        const int slots = sm_count * tc_ctas_per_sm(p);
        const int tiles = (npages + 1) / 2;
        if (npages == 0) {
            pl.splits_q = 0;
            pl.pages_per_split = 2;
        } else {
            int want = slots / units;
            if (want < 1) want = 1;
            if (want > tiles) want = tiles;
            int tps = (tiles + want - 1) / want;
            if (tps > 16) tps = 16;                     // the kernel keeps a split's scores on chip
            pl.pages_per_split = 2 * tps;
            if (pl.pages_per_split > 256) pl.pages_per_split = 256;   // page ids staged in shared memory
            pl.splits_q = (npages + pl.pages_per_split - 1) / pl.pages_per_split;
        }
        pl.grid_x = pl.window_split + pl.splits_q;
        if (pl.grid_x == 0) pl.grid_x = 1;              // all-empty: one CTA writes zeros
        pl.window_slot = pl.splits_q;                   // first window slot
        pl.total_splits = pl.grid_x;
        return pl;
    }
    // about four resident CTAs per SM over the quantized pages
    int want = (4 * sm_count + units - 1) / units;
    if (want < 1) want = 1;
    if (npages == 0) {
        pl.splits_q = 0;
        pl.pages_per_split = 1;
    } else {
        if (want > npages) want = npages;
        pl.pages_per_split = (npages + want - 1) / want;
        pl.splits_q = (npages + pl.pages_per_split - 1) / pl.pages_per_split;
    }
    pl.total_splits = pl.splits_q + pl.window_split;
    if (pl.total_splits == 0) pl.total_splits = 1;   // all-empty: one split writes zeros
    pl.grid_x = pl.total_splits;
    pl.window_slot = pl.total_splits - 1;
    return pl;
}

size_t decode_workspace_bytes(const Params& p, int batch, const DecodePlan& pl) {
    if (pl.mma) return mma_workspace_layout(p, batch, pl.ctas, nullptr);
    size_t rows = size_t(batch) * p.hq * pl.total_splits;
    size_t o = rows * p.d * sizeof(float);
    o = (o + 255) & ~size_t(255);
    return o + rows * 2 * sizeof(float);
}

namespace {

constexpr unsigned FULL = 0xffffffffu;

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

// grid (total_splits, Hkv, B), 128 threads.  Split s < splits_q covers
// quantized pages [s*pps, (s+1)*pps); the last split (when the layout has a
// window) covers the bf16 window.  Each split writes, per query head, the
// unnormalised output o, the running max m (log2 domain) and the sum l.
template <int D, int KB, int VB>
__global__ void __launch_bounds__(128) decode_split_simt(Params p, const void* __restrict__ q, int q_bf16,
                                                         const int32_t* __restrict__ lens, int max_len,
                                                         float scale_log2, float* __restrict__ ws_o,
                                                         float* __restrict__ ws_ml, DecodePlan pl) {
    constexpr int KW = D * KB / 32;            // words per key row
    constexpr int KPW = 32 / KB;               // key codes per word
    constexpr int VW = kPage * VB / 32;        // words per value channel row (one page)
    constexpr int VPW = 32 / VB;
    constexpr int NVG_MAX = D / 16;
    __shared__ float q_s[kMaxGqa][D];
    __shared__ float qsum_s[kMaxGqa][D / 16];
    __shared__ float s_s[kMaxGqa][kPage];
    __shared__ float pv_s[kMaxGqa][NVG_MAX][kPage];
    __shared__ float m_s[kMaxGqa], l_s[kMaxGqa], a_s[kMaxGqa];
    __shared__ float pz_s[kMaxGqa][NVG_MAX];

    const int b = blockIdx.z, h = blockIdx.y, split = blockIdx.x;
    const int g = p.g, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = max(0, min(lens[b], max_len));
    const int Lq = max(0, L - p.W);
    const bool is_win = pl.window_split && split == pl.total_splits - 1;
    int c_begin, c_end;                        // token range [c_begin, c_end)
    if (is_win) {
        c_begin = Lq;
        c_end = L;
    } else {
        c_begin = split * pl.pages_per_split * kPage;
        c_end = min(Lq, (split + 1) * pl.pages_per_split * kPage);
    }
    const size_t row0 = (size_t(b) * p.hq + size_t(h) * g) * pl.total_splits + split;
    if (c_begin >= c_end) {
        for (int i = tid; i < g * D; i += blockDim.x)
            ws_o[(row0 + size_t(i / D) * pl.total_splits) * D + (i % D)] = 0.0f;
        if (tid < g) {
            ws_ml[(row0 + size_t(tid) * pl.total_splits) * 2 + 0] = -INFINITY;
            ws_ml[(row0 + size_t(tid) * pl.total_splits) * 2 + 1] = 0.0f;
        }
        return;
    }

    // query rows of this kv-group, fp32; rotated for quantized keys
    for (int i = tid; i < g * D; i += blockDim.x) {
        size_t off = (size_t(b) * p.hq + size_t(h) * g + i / D) * D + (i % D);
        q_s[i / D][i % D] = q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[off])
                                   : reinterpret_cast<const float*>(q)[off];
    }
    __syncthreads();
    if (!is_win && p.rotate) {
        for (int r = warp; r < g; r += 4) {
            float x[D / 32];
#pragma unroll
            for (int i = 0; i < D / 32; ++i) x[i] = q_s[r][lane * (D / 32) + i];
            rotate_warp<D>(x, p.signs, lane);
#pragma unroll
            for (int i = 0; i < D / 32; ++i) q_s[r][lane * (D / 32) + i] = x[i];
        }
        __syncthreads();
    }
    if (!is_win) {
        for (int i = tid; i < g * p.nkg; i += blockDim.x) {
            const int r = i / p.nkg, grp = i % p.nkg;
            float s = 0.0f;
            for (int j = grp * p.kg; j < (grp + 1) * p.kg; ++j) s += q_s[r][j];
            qsum_s[r][grp] = s;
        }
    }
    if (tid < g) {
        m_s[tid] = -INFINITY;
        l_s[tid] = 0.0f;
        for (int v = 0; v < NVG_MAX; ++v) pz_s[tid][v] = 0.0f;
    }
    __syncthreads();

    const int t = tid & (kPage - 1), hp = tid >> 6;     // score phase: token, head parity
    const int jc = (D == 128) ? tid : (tid & 63);         // value phase: channel
    const int hsel = (D == 128) ? 0 : (tid >> 6);
    const int hstep = (D == 128) ? 1 : 2;
    const int vgrp_j = jc / p.vg;
    float o[kMaxGqa];
#pragma unroll
    for (int r = 0; r < kMaxGqa; ++r) o[r] = 0.0f;

    for (int cb = c_begin; cb < c_end; cb += kPage) {
        const int chunk_base = is_win ? cb : (cb & ~(kPage - 1));
        const int pos = chunk_base + t;
        const bool valid = pos >= c_begin && pos < c_end;
        int page = -1;
        if (!is_win) page = phys_page(p, b, chunk_base / kPage);
        // ---------------- scores
        if (is_win) {
            float acc[kMaxGqa / 2];
#pragma unroll
            for (int r = 0; r < kMaxGqa / 2; ++r) acc[r] = 0.0f;
            if (valid) {
                const __nv_bfloat16* kr = p.k_win + win_off(p, b, h, pos);
                for (int j = 0; j < D; j += 2) {
                    float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kr + j));
#pragma unroll
                    for (int r = 0; r < kMaxGqa / 2; ++r) {
                        const int hh = hp + 2 * r;
                        if (hh < g) acc[r] = fmaf(kv.y, q_s[hh][j + 1], fmaf(kv.x, q_s[hh][j], acc[r]));
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < kMaxGqa / 2; ++r) {
                const int hh = hp + 2 * r;
                if (hh < g) s_s[hh][t] = valid ? acc[r] * scale_log2 : -INFINITY;
            }
        } else {
            const bool ok = valid && page >= 0;
            uint32_t kw[KW];
            float2 km[D / 16];
            if (ok) {
#pragma unroll
                for (int w = 0; w < KW; ++w) kw[w] = *k_word(p, page, h, pos % kPage, w);
                const uint32_t* mr = k_meta_row(p, page, h, pos % kPage);
                for (int gi = 0; gi < p.nkg; ++gi) km[gi] = meta_f2(mr[gi]);
            }
#pragma unroll
            for (int r = 0; r < kMaxGqa / 2; ++r) {
                const int hh = hp + 2 * r;
                if (hh >= g) continue;
                float acc = 0.0f;
                if (ok) {
                    float dot = 0.0f;
#pragma unroll
                    for (int j = 0; j < D; ++j) {
                        const float c = (float)((kw[j / KPW] >> (KB * (j % KPW))) & ((1u << KB) - 1u));
                        dot = fmaf(c, q_s[hh][j], dot);
                        if ((j + 1) % 16 == 0 && ((j + 1) % p.kg) == 0) {
                            const int gi = j / p.kg;
                            acc = fmaf(km[gi].x, dot, fmaf(km[gi].y, qsum_s[hh][gi], acc));
                            dot = 0.0f;
                        }
                    }
                }
                s_s[hh][t] = ok ? acc * scale_log2 : -INFINITY;
            }
        }
        __syncthreads();
        // ---------------- online softmax: warp w owns heads w, w+4
        for (int r = warp; r < g; r += 4) {
            const float s0 = s_s[r][lane], s1 = s_s[r][lane + 32];
            const float m_old = m_s[r];
            const float m_new = fmaxf(m_old, warp_max(fmaxf(s0, s1)));
            const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
            const float alpha = exp2f(m_old - m_use);
            const float p0 = exp2f(s0 - m_use), p1 = exp2f(s1 - m_use);
            const float lsum = warp_sum(p0 + p1);
            if (is_win) {
                pv_s[r][0][lane] = p0;
                pv_s[r][0][lane + 32] = p1;
            } else {
                const int pos0 = chunk_base + lane, pos1 = chunk_base + lane + 32;
                const bool ok0 = page >= 0 && pos0 >= c_begin && pos0 < c_end;
                const bool ok1 = page >= 0 && pos1 >= c_begin && pos1 < c_end;
                for (int v = 0; v < p.nvg; ++v) {
                    float2 m0 = ok0 ? meta_f2(v_meta_row(p, page, h, lane)[v]) : make_float2(0.f, 0.f);
                    float2 m1 = ok1 ? meta_f2(v_meta_row(p, page, h, lane + 32)[v]) : make_float2(0.f, 0.f);
                    pv_s[r][v][lane] = p0 * m0.x;
                    pv_s[r][v][lane + 32] = p1 * m1.x;
                    const float z = warp_sum(p0 * m0.y + p1 * m1.y);
                    if (lane == 0) pz_s[r][v] = fmaf(pz_s[r][v], alpha, z);
                }
            }
            if (lane == 0) {
                m_s[r] = m_new;
                l_s[r] = fmaf(l_s[r], alpha, lsum);
                a_s[r] = alpha;
            }
        }
        __syncthreads();
        // ---------------- values
        if (is_win) {
            for (int r = hsel; r < g; r += hstep) o[r] *= a_s[r];
            const int n = min(kPage, c_end - chunk_base);
            int tt = 0;
            for (; tt + 16 <= n; tt += 16) {               // 16 independent loads in flight
                float v[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    v[k] = __bfloat162float(p.v_win[win_off(p, b, h, chunk_base + tt + k) + jc]);
#pragma unroll
                for (int k = 0; k < 16; ++k)
#pragma unroll
                    for (int r = 0; r < kMaxGqa; ++r)
                        if (r < g && (r - hsel) % hstep == 0 && r >= hsel)
                            o[r] = fmaf(pv_s[r][0][tt + k], v[k], o[r]);
            }
            for (; tt < n; ++tt) {
                const float v = __bfloat162float(p.v_win[win_off(p, b, h, chunk_base + tt) + jc]);
#pragma unroll
                for (int r = 0; r < kMaxGqa; ++r)
                    if (r < g && (r - hsel) % hstep == 0 && r >= hsel) o[r] = fmaf(pv_s[r][0][tt], v, o[r]);
            }
        } else {
            uint32_t vw[VW];
            if (page >= 0) {
#pragma unroll
                for (int w = 0; w < VW; ++w) vw[w] = *v_word(p, page, h, jc, w);
            }
#pragma unroll
            for (int r = 0; r < kMaxGqa; ++r) {
                if (r >= g || r < hsel || (r - hsel) % hstep) continue;
                float acc = o[r] * a_s[r];
                if (page >= 0) {
#pragma unroll 16
                    for (int tt = 0; tt < kPage; ++tt) {
                        const float c = (float)((vw[tt / VPW] >> (VB * (tt % VPW))) & ((1u << VB) - 1u));
                        acc = fmaf(pv_s[r][vgrp_j][tt], c, acc);
                    }
                }
                o[r] = acc;
            }
        }
        __syncthreads();
    }
    // partial results of this split
#pragma unroll
    for (int r = 0; r < kMaxGqa; ++r) {
        if (r >= g || r < hsel || (r - hsel) % hstep) continue;
        const float extra = is_win ? 0.0f : pz_s[r][vgrp_j];
        ws_o[(row0 + size_t(r) * pl.total_splits) * D + jc] = o[r] + extra;
    }
    if (tid < g) {
        ws_ml[(row0 + size_t(tid) * pl.total_splits) * 2 + 0] = m_s[tid];
        ws_ml[(row0 + size_t(tid) * pl.total_splits) * 2 + 1] = l_s[tid];
    }
}

// one warp per (sequence, query head): merge the splits' (m, l, o)
template <int D>
__global__ void __launch_bounds__(128) combine_kernel(int rows, int S, const float* __restrict__ ws_o,
                                                      const float* __restrict__ ws_ml, float* __restrict__ out,
                                                      float* __restrict__ lse) {
    constexpr int CPL = D / 32;
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31;
    const float* ml = ws_ml + size_t(row) * S * 2;
    float M = -INFINITY;
    for (int s = lane; s < S; s += 32) M = fmaxf(M, ml[2 * s]);
    M = warp_max(M);
    float acc[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] = 0.0f;
    float lsum = 0.0f;
    if (M != -INFINITY) {
        // four splits per round, every load of the round issued before use;
        // a split with m = -inf (no positions) has o = 0 and weight 0
        for (int s0 = 0; s0 < S; s0 += 4) {
            float mv[4], lv[4], ov[4][CPL];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const bool in = s0 + u < S;
                mv[u] = in ? ml[2 * (s0 + u)] : -INFINITY;
                lv[u] = in ? ml[2 * (s0 + u) + 1] : 0.0f;
                const float* os = ws_o + (size_t(row) * S + (in ? s0 + u : 0)) * D + lane * CPL;
#pragma unroll
                for (int i = 0; i < CPL; ++i) ov[u][i] = in ? os[i] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float w = (mv[u] == -INFINITY) ? 0.0f : exp2f(mv[u] - M);
                lsum = fmaf(lv[u], w, lsum);
#pragma unroll
                for (int i = 0; i < CPL; ++i) acc[i] = fmaf(ov[u][i], w, acc[i]);
            }
        }
    }
    float* o = out + size_t(row) * D + lane * CPL;
    const float inv = (lsum > 0.0f) ? 1.0f / lsum : 0.0f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) o[i] = acc[i] * inv;
    if (lse && lane == 0) lse[row] = (lsum > 0.0f) ? (M + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
}

template <int D, int KB, int VB>
cudaError_t launch_simt(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                        float scale_log2, float* ws_o, float* ws_ml, const DecodePlan& pl, cudaStream_t s) {
    dim3 grid(pl.total_splits, p.hkv, p.batch);
    decode_split_simt<D, KB, VB><<<grid, 128, 0, s>>>(p, q, q_bf16, lens, max_len, scale_log2, ws_o, ws_ml, pl);
    return cudaGetLastError();
}

template <int D, int KB>
cudaError_t dispatch_vb(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                        float sl2, float* wo, float* wml, const DecodePlan& pl, cudaStream_t s) {
    switch (p.vb) {
        case 1: return launch_simt<D, KB, 1>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 2: return launch_simt<D, KB, 2>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 4: return launch_simt<D, KB, 4>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        default: return launch_simt<D, KB, 8>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
    }
}

template <int D>
cudaError_t dispatch_kb(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                        float sl2, float* wo, float* wml, const DecodePlan& pl, cudaStream_t s) {
    switch (p.kb) {
        case 1: return dispatch_vb<D, 1>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 2: return dispatch_vb<D, 2>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        case 4: return dispatch_vb<D, 4>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
        default: return dispatch_vb<D, 8>(p, q, q_bf16, lens, max_len, sl2, wo, wml, pl, s);
    }
}

}  // namespace

// decode diagnostics: [0] expired bounded waits, [1] tickets above their count
__device__ unsigned int g_decode_status[2];

namespace {
constexpr int kMaxDev = 64;
unsigned* g_status_addr[kMaxDev];
unsigned* status_ptr() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
    if (!g_status_addr[dev]) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_decode_status) != cudaSuccess) return nullptr;
        g_status_addr[dev] = static_cast<unsigned*>(a);
    }
    return g_status_addr[dev];
}
}  // namespace

cudaError_t decode_status(unsigned* wait_timeouts, unsigned* bad_tickets, bool clear) {
    unsigned v[2] = {0u, 0u};
    cudaError_t e = cudaMemcpyFromSymbol(v, g_decode_status, sizeof(v));
    if (e != cudaSuccess) return e;
    if (wait_timeouts) *wait_timeouts = v[0];
    if (bad_tickets) *bad_tickets = v[1];
    if (clear) {
        const unsigned z[2] = {0u, 0u};
        e = cudaMemcpyToSymbol(g_decode_status, z, sizeof(z));
    }
    return e;
}

cudaError_t launch_decode(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                          float sm_scale, float* out, float* lse, void* ws, const DecodePlan& pl,
                          cudaStream_t s) {
    if (p.batch <= 0) return cudaSuccess;
    unsigned* status = status_ptr();
    if (!status) return cudaErrorInvalidSymbol;
    const size_t rows = size_t(p.batch) * p.hq;
    float* ws_o = reinterpret_cast<float*>(ws);
    size_t ob = (rows * pl.total_splits * p.d * sizeof(float) + 255) & ~size_t(255);
    float* ws_ml = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + ob);
    const float sl2 = sm_scale * 1.4426950408889634f;
    if (pl.mma) {
        size_t off_tickets = 0;
        mma_workspace_layout(p, p.batch, pl.ctas, &off_tickets);
        float* part = reinterpret_cast<float*>(ws);
        uint32_t* tickets = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + off_tickets);
        switch (p.kb) {
            case 1: return launch_decode_mma_k1(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, pl.ctas, pl.after_append, status, s);
            case 2: return launch_decode_mma_k2(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, pl.ctas, pl.after_append, status, s);
            case 4: return launch_decode_mma_k4(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, pl.ctas, pl.after_append, status, s);
            default: return launch_decode_mma_k8(p, q, q_bf16, lens, max_len, sl2, out, lse, part, tickets, pl.ctas, pl.after_append, status, s);
        }
    }
    cudaError_t e = pl.tc ? launch_decode_tc(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, status, s)
                  : (p.d == 128) ? dispatch_kb<128>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, s)
                                 : dispatch_kb<64>(p, q, q_bf16, lens, max_len, sl2, ws_o, ws_ml, pl, s);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((rows + 3) / 4));
    if (p.d == 128) combine_kernel<128><<<grid, 128, 0, s>>>((int)rows, pl.total_splits, ws_o, ws_ml, out, lse);
    else combine_kernel<64><<<grid, 128, 0, s>>>((int)rows, pl.total_splits, ws_o, ws_ml, out, lse);
    return cudaGetLastError();
}

}  // namespace kvq

// Decode attention (one query token per sequence) over a cache whose key
// groups run along positions of one channel ("Granularitas kuantisasi ...":
// the grouping axis may run along token positions), head_dim 128.
//
// What it computes is the decode of "Kuantisasi KV cache mengganggu
// attention ..." (s = q K^T * sm_scale, a = softmax(s), o = a V) over the
// cache as it holds the positions: pages below Q = kg*floor(max(0, L-W)/kg),
// the bf16 ring (W + kg - 1 slots) above.  With the scale and zero point of
// a key group constant over its kg positions of one channel, the query
// absorbs them: for a position t of key group gi,
//     q . k^_t = sum_j (q_j scale_{gi,j}) c_{t,j} + sum_j q_j zero_{gi,j},
// so a group's scores are one dot product of the codes with q' = q*scale,
// plus a constant b.  Values keep per-token groups: o = sum_t (p_t vscale_t)
// c_t + sum_t p_t vzero_t per value group.
//
// One CTA of 512 threads per (sequence, kv-head), all g query heads of the
// kv-group together.  Per 64-position page: the page's raw blocks (key codes,
// key metadata, value codes, value metadata) are copied into shared memory
// one page ahead with cp.async; q' and b are formed per key group; scores
// by (position, 16-channel part) threads reduced with shuffles; online
// softmax per head (log2 domain); the weighted value codes by (channel,
// position quarter) threads.  Ring positions are read as bf16 rows.  CUDA
// cores only: the work per byte is a few multiply-adds.
#include <cuda_fp16.h>

#include "kvq_internal.cuh"
#include "kvq_tc_ptx.cuh"

namespace kvq {
namespace {

constexpr int PD = 128;
constexpr int PT = 64;              // positions per page
constexpr int PTH = 512;            // threads per CTA
constexpr int GMAX = 8;             // query heads per kv-head (kernels for up to 4 and up to 8)
constexpr unsigned FULLM = 0xffffffffu;

// one stage of raw page data: key codes [d][kchan], key metadata [64/kg][d],
// value codes [d][vchan], value metadata [64][nvg] (byte sizes for 8-bit codes,
// 16-position key groups, 16-channel value groups at most)
constexpr int ST_KC = PD * 64;
constexpr int ST_KM = (PT / 16) * PD * 4;
constexpr int ST_VC = PD * 64;
constexpr int ST_VM = PT * 8 * 4;
constexpr int ST_BYTES = ST_KC + ST_KM + ST_VC + ST_VM;

template <int NH>
struct PcSmem {
    float q[PD][NH];                // the query (sm_scale * log2 e folded in), heads innermost
    float qp[4][PD][NH];            // q * key scale, per key group of the page
    float qb[4][NH];                // sum_j q_j * key zero, per key group
    float s[PT][NH];                // scores, then weights
    float pv[8][PT][NH];            // weight * value scale, per value group
    float pz[8][NH];                // sum_t weight * value zero, per value group
    float m[NH], l[NH], alpha[NH];
    __align__(16) uint8_t raw[2][ST_BYTES];
    int pages[1];                   // page ids of the sequence's pages (grows into the dynamic tail)
};

__device__ __forceinline__ float hbits(uint32_t b) {
    __half_raw r;
    r.x = uint16_t(b);
    return __half2float(__half(r));
}
__device__ __forceinline__ float bfbits(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ void cpa16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cpa_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cpa_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// code of position slot t (0..63) in a channel run of BITS*8 bytes stored
// chunk-major above 16 bytes: [chunk][d][min(16, run)] (run of channel j)
template <int BITS>
__device__ __forceinline__ uint32_t run_code(const uint8_t* base, int j, int t) {
    constexpr int chan = PT * BITS / 8, cw = chan < 16 ? chan : 16;
    const int bit = t * BITS, byte = bit >> 3;
    const uint8_t c8 = base[(byte / cw) * (PD * cw) + j * cw + (byte % cw)];
    return (uint32_t(c8) >> (bit & 7)) & ((1u << BITS) - 1u);
}
// the codes of positions 16 qt .. 16 qt + 15 of channel j's run, as 16*BITS bits
template <int BITS>
__device__ __forceinline__ void run_quarter(const uint8_t* base, int j, int qt, uint32_t (&w)[4]) {
    constexpr int chan = PT * BITS / 8, cw = chan < 16 ? chan : 16;
    const int byte = 2 * BITS * qt;                 // first byte of the quarter
    const uint8_t* a = base + (byte / cw) * (PD * cw) + j * cw + (byte % cw);
    if constexpr (BITS == 1) {
        w[0] = *reinterpret_cast<const uint16_t*>(a);
    } else if constexpr (BITS == 2) {
        w[0] = *reinterpret_cast<const uint32_t*>(a);
    } else if constexpr (BITS == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(a);
        w[0] = u.x, w[1] = u.y;
    } else {
        const uint4 u = *reinterpret_cast<const uint4*>(a);
        w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
    }
}

template <int NH>
__device__ __forceinline__ void ld_heads(const float* a, float (&x)[NH]) {
#pragma unroll
    for (int r = 0; r < NH; r += 4) {
        const float4 v = *reinterpret_cast<const float4*>(a + r);
        x[r] = v.x, x[r + 1] = v.y, x[r + 2] = v.z, x[r + 3] = v.w;
    }
}

template <int KB, int VB, int NH>
__global__ void __launch_bounds__(PTH, 1) decode_pc_kernel(const Params p, const void* __restrict__ qv, int q_bf16,
                                                           const int32_t* __restrict__ lens, int max_len,
                                                           float sl2, float* __restrict__ out,
                                                           float* __restrict__ lse) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    PcSmem<NH>& sm = *reinterpret_cast<PcSmem<NH>*>(smem_raw);
    const int h = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = p.g, kg = p.kg, nkg_page = PT / kg, vg = p.vg, nvg = p.nvg;
    const int L = max(0, min(lens[b], max_len));
    const size_t orow0 = size_t(b) * p.hq + size_t(h) * g;
    if (L == 0) {                                   // an empty sequence: o = 0, lse = -inf
        for (int e = tid; e < g * PD; e += PTH) {
            out[(orow0 + e / PD) * PD + e % PD] = 0.0f;
            if (lse && e % PD == 0) lse[orow0 + e / PD] = -INFINITY;
        }
        return;
    }
    const int R = p.W + kg - 1;                     // ring slots
    const int Q = L - p.W > 0 ? ((L - p.W) / kg) * kg : 0;   // positions below Q live in pages
    constexpr int kchan = PT * KB / 8, vchan = PT * VB / 8;
    const int KC = PD * kchan, KM = nkg_page * PD * 4, VC = PD * vchan, VM = PT * nvg * 4;
    const int ntiles = (L + PT - 1) / PT;
    const size_t blk = size_t(h);

    // ---- the query of the g heads (zeros for heads r >= g)
    for (int e = tid; e < NH * PD; e += PTH) {
        const int r = e / PD, j = e % PD;
        float x = 0.0f;
        if (r < g) {
            const size_t idx = (orow0 + r) * PD + j;
            x = q_bf16 ? bfbits(static_cast<const uint16_t*>(qv)[idx]) : static_cast<const float*>(qv)[idx];
        }
        sm.q[j][r] = x * sl2;
    }
    if (tid < NH) {
        sm.m[tid] = -INFINITY;
        sm.l[tid] = 0.0f;
    }
    // page ids of the quantized tiles, read once (not one global load per tile)
    const int npq = (Q + PT - 1) / PT;
    for (int i = tid; i < npq; i += PTH) {
        const int pg = i < p.max_pages ? p.page_table[size_t(b) * p.max_pages + i] : -1;
        sm.pages[i] = pg >= p.num_pages ? -1 : pg;
    }
    __syncthreads();

    // raw page blocks of tile i into stage i % 2 (zeros for an unmapped page)
    auto stage = [&](int i) {
        if (i >= ntiles || i * PT >= Q) return;
        uint8_t* dst = sm.raw[i & 1];
        const int pg = sm.pages[i];
        const int n16 = (KC + KM + VC + VM) / 16;
        for (int c = tid; c < n16; c += PTH) {
            const int off = 16 * c;
            uint8_t* d = dst + off;
            if (pg < 0) {
                *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
                continue;
            }
            const uint8_t* src;
            if (off < KC) src = p.k_codes + (size_t(pg) * p.hkv + blk) * KC + off;
            else if (off < KC + KM)
                src = reinterpret_cast<const uint8_t*>(p.k_meta) + (size_t(pg) * p.hkv + blk) * KM + (off - KC);
            else if (off < KC + KM + VC) src = p.v_codes + (size_t(pg) * p.hkv + blk) * VC + (off - KC - KM);
            else
                src = reinterpret_cast<const uint8_t*>(p.v_meta) + (size_t(pg) * p.hkv + blk) * VM +
                      (off - KC - KM - VC);
            cpa16(ptx::smem_u32(d), src);
        }
    };
    stage(0);
    cpa_commit();

    float o_acc[NH];                                 // lanes with quarter 0: channel vj, every head
#pragma unroll
    for (int r = 0; r < NH; ++r) o_acc[r] = 0.0f;
    // (channel, quarter) of the value threads
    const int vj = warp * 8 + (lane >> 2), vq = lane & 3;
    // (position, part) of the score threads; a part is channels sp, sp + 8, ..., sp + 120
    const int st = warp * 4 + (lane >> 3), sp = lane & 7;

    for (int i = 0; i < ntiles; ++i) {
        stage(i + 1);
        cpa_commit();
        cpa_wait_1();
        __syncthreads();                             // stage i landed for every thread
        const int t0 = i * PT;
        const uint8_t* raw = sm.raw[i & 1];
        const uint8_t* kc = raw;
        const uint32_t* km = reinterpret_cast<const uint32_t*>(raw + KC);
        const uint8_t* vc = raw + KC + KM;
        const uint32_t* vm = reinterpret_cast<const uint32_t*>(raw + KC + KM + VC);
        const bool paged_any = t0 < Q;

        // ---- q' = q * key scale and b = q . key zero, per key group of the page
        if (paged_any) {
            for (int e = tid; e < nkg_page * PD; e += PTH) {
                const int gi = e / PD, j = e % PD;
                const float sc = hbits(km[gi * PD + j] & 0xffffu);
#pragma unroll
                for (int r = 0; r < NH; ++r) sm.qp[gi][j][r] = sm.q[j][r] * sc;
            }
            // one warp per key group: 4 channels per lane, then a warp sum per head
            for (int gi = warp; gi < nkg_page; gi += PTH / 32) {
                float acc[NH];
#pragma unroll
                for (int r = 0; r < NH; ++r) acc[r] = 0.0f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int j = 4 * lane + c;
                    const float z = hbits(km[gi * PD + j] >> 16);
#pragma unroll
                    for (int r = 0; r < NH; ++r) acc[r] = fmaf(sm.q[j][r], z, acc[r]);
                }
#pragma unroll
                for (int r = 0; r < NH; ++r) {
#pragma unroll
                    for (int o = 16; o; o >>= 1) acc[r] += __shfl_xor_sync(FULLM, acc[r], o);
                    if (lane == 0) sm.qb[gi][r] = acc[r];
                }
            }
        }
        __syncthreads();

        // ---- scores: thread (position st, channels sp + 8c), every head
        {
            const int pos = t0 + st;
            float acc[NH];
#pragma unroll
            for (int r = 0; r < NH; ++r) acc[r] = 0.0f;
            if (pos < L) {
                if (pos < Q) {
                    const int gi = st / kg;
#pragma unroll 4
                    for (int c = 0; c < 16; ++c) {
                        const int j = sp + 8 * c;
                        const float x = float(run_code<KB>(kc, j, st));
                        float qq[NH];
                        ld_heads<NH>(&sm.qp[gi][j][0], qq);
#pragma unroll
                        for (int r = 0; r < NH; ++r) acc[r] = fmaf(qq[r], x, acc[r]);
                    }
                } else {
                    const uint16_t* kw = reinterpret_cast<const uint16_t*>(p.k_win) +
                                         ((size_t(b) * p.hkv + blk) * R + size_t(pos % R)) * PD;
#pragma unroll 4
                    for (int c = 0; c < 16; ++c) {
                        const int j = sp + 8 * c;
                        const float x = bfbits(kw[j]);
                        float qq[NH];
                        ld_heads<NH>(&sm.q[j][0], qq);
#pragma unroll
                        for (int r = 0; r < NH; ++r) acc[r] = fmaf(qq[r], x, acc[r]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                float v = acc[r];
                v += __shfl_xor_sync(FULLM, v, 1);
                v += __shfl_xor_sync(FULLM, v, 2);
                v += __shfl_xor_sync(FULLM, v, 4);
                acc[r] = v;
            }
            if (sp == 0) {
#pragma unroll
                for (int r = 0; r < NH; ++r)
                    sm.s[st][r] = pos >= L ? -INFINITY : (pos < Q ? acc[r] + sm.qb[st / kg][r] : acc[r]);
            }
        }
        __syncthreads();

        // ---- online softmax: warp r for head r
        if (warp < g) {
            const int r = warp;
            const float x0 = sm.s[lane][r], x1 = sm.s[lane + 32][r];
            float mx = fmaxf(x0, x1);
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULLM, mx, o));
            const float m_old = sm.m[r];
            const float mn = fmaxf(m_old, mx);       // finite: position t0 < L is in every tile
            const float p0 = exp2f(x0 - mn), p1 = exp2f(x1 - mn);
            float sum = p0 + p1;
#pragma unroll
            for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(FULLM, sum, o);
            const float al = exp2f(m_old - mn);      // 0 on the first tile
            sm.s[lane][r] = p0;
            sm.s[lane + 32][r] = p1;
            if (lane == 0) {
                sm.m[r] = mn;
                sm.l[r] = fmaf(sm.l[r], al, sum);
                sm.alpha[r] = al;
            }
        } else if (warp < NH && lane < PT / 2) {
            // heads r >= g: zero weights (their rows are never output)
            sm.s[lane][warp] = 0.0f;
            sm.s[lane + 32][warp] = 0.0f;
            if (lane == 0) sm.alpha[warp] = 0.0f;
        }
        __syncthreads();

        // ---- weights times value scale, and the zero-point sums, per value group
        if (paged_any) {
            for (int e = tid; e < nvg * PT; e += PTH) {
                const int gv = e / PT, t = e % PT;
                const float sc = t0 + t < Q ? hbits(vm[t * nvg + gv] & 0xffffu) : 0.0f;
#pragma unroll
                for (int r = 0; r < NH; ++r) sm.pv[gv][t][r] = sm.s[t][r] * sc;
            }
            for (int gv = warp; gv < nvg; gv += PTH / 32) {
                float acc[NH];
#pragma unroll
                for (int r = 0; r < NH; ++r) acc[r] = 0.0f;
                for (int t = lane; t < PT; t += 32) {
                    const float z = t0 + t < Q ? hbits(vm[t * nvg + gv] >> 16) : 0.0f;
#pragma unroll
                    for (int r = 0; r < NH; ++r) acc[r] = fmaf(sm.s[t][r], z, acc[r]);
                }
#pragma unroll
                for (int r = 0; r < NH; ++r) {
#pragma unroll
                    for (int o = 16; o; o >>= 1) acc[r] += __shfl_xor_sync(FULLM, acc[r], o);
                    if (lane == 0) sm.pz[gv][r] = acc[r];
                }
            }
        }
        __syncthreads();

        // ---- o = o * alpha + sum_t w_t v_t: thread (channel vj, positions 16 vq .. 16 vq + 15)
        {
            float acc[NH];
#pragma unroll
            for (int r = 0; r < NH; ++r) acc[r] = 0.0f;
            const int gv = vj / vg;
            const int tq0 = t0 + 16 * vq;
            if (tq0 + 15 < Q) {
                // every position of the quarter in the page: codes from one load
                uint32_t w[4];
                run_quarter<VB>(vc, vj, vq, w);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int bit = c * VB;
                    const float x = float((w[bit >> 5] >> (bit & 31)) & ((1u << VB) - 1u));
                    float pw[NH];
                    ld_heads<NH>(&sm.pv[gv][16 * vq + c][0], pw);
#pragma unroll
                    for (int r = 0; r < NH; ++r) acc[r] = fmaf(pw[r], x, acc[r]);
                }
            } else {
                for (int c = 0; c < 16; ++c) {
                    const int t = 16 * vq + c, pos = t0 + t;
                    if (pos >= L) break;
                    float x;
                    float pw[NH];
                    if (pos < Q) {
                        x = float(run_code<VB>(vc, vj, t));
                        ld_heads<NH>(&sm.pv[gv][t][0], pw);
                    } else {
                        x = bfbits(reinterpret_cast<const uint16_t*>(
                            p.v_win)[((size_t(b) * p.hkv + blk) * R + size_t(pos % R)) * PD + vj]);
                        ld_heads<NH>(&sm.s[t][0], pw);
                    }
#pragma unroll
                    for (int r = 0; r < NH; ++r) acc[r] = fmaf(pw[r], x, acc[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                float v = acc[r];
                v += __shfl_xor_sync(FULLM, v, 1);
                v += __shfl_xor_sync(FULLM, v, 2);
                if (vq == 0) o_acc[r] = fmaf(o_acc[r], sm.alpha[r], v + (paged_any ? sm.pz[gv][r] : 0.0f));
            }
        }
        __syncthreads();                             // stage i is free for tile i + 2
    }
    cpa_wait_0();

    // ---- o / l, lse = (m + log2 l) ln 2
    if (vq == 0) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            if (r >= g) break;
            const float l = sm.l[r];
            out[(orow0 + r) * PD + vj] = o_acc[r] / l;
            if (lse && vj == 0) lse[orow0 + r] = (sm.m[r] + log2f(l)) * 0.693147180559945309f;
        }
    }
}

template <int KB, int NH>
cudaError_t launch_nh_pc(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                         float* out, float* lse, cudaStream_t s) {
    const dim3 grid(p.hkv, p.batch);
    // the page-id table grows past the struct: one int per quantized page
    const int bytes = int(sizeof(PcSmem<NH>)) + 4 * (max_len / PT + 1);
    auto go = [&](auto kern) -> cudaError_t {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        kern<<<grid, PTH, bytes, s>>>(p, q, q_bf16, lens, max_len, sl2, out, lse);
        return cudaGetLastError();
    };
    switch (p.vb) {
        case 1: return go(decode_pc_kernel<KB, 1, NH>);
        case 2: return go(decode_pc_kernel<KB, 2, NH>);
        case 4: return go(decode_pc_kernel<KB, 4, NH>);
        default: return go(decode_pc_kernel<KB, 8, NH>);
    }
}

template <int KB>
cudaError_t launch_kb_pc(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                         float* out, float* lse, cudaStream_t s) {
    if (p.g <= 4) return launch_nh_pc<KB, 4>(p, q, q_bf16, lens, max_len, sl2, out, lse, s);
    return launch_nh_pc<KB, 8>(p, q, q_bf16, lens, max_len, sl2, out, lse, s);
}

}  // namespace

bool decode_pc_supported(const Params& p, int max_len) {
    // shared memory: the struct plus one page id per quantized page
    const size_t bytes = sizeof(PcSmem<8>) + 4 * size_t(max_len / PT + 1);
    return p.d == PD && p.g >= 1 && p.g <= GMAX && (p.kg == 16 || p.kg == 32 || p.kg == 64) && p.vg >= 16 &&
           PD % p.vg == 0 && !p.rotate && bytes <= 227 * 1024;
}

cudaError_t launch_decode_per_channel(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                                      float sm_scale, float* out, float* lse, cudaStream_t s) {
    const float sl2 = sm_scale * 1.4426950408889634f;
    switch (p.kb) {
        case 1: return launch_kb_pc<1>(p, q, q_bf16, lens, max_len, sl2, out, lse, s);
        case 2: return launch_kb_pc<2>(p, q, q_bf16, lens, max_len, sl2, out, lse, s);
        case 4: return launch_kb_pc<4>(p, q, q_bf16, lens, max_len, sl2, out, lse, s);
        default: return launch_kb_pc<8>(p, q, q_bf16, lens, max_len, sl2, out, lse, s);
    }
}

}  // namespace kvq

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
// One CTA per (sequence, kv-head), all g query heads of the kv-group
// together; its warps (up to 8) take the pair's 64-position tiles in turn (warp w:
// tiles w, w + NW, ...), each warp on its own: the raw page blocks (key
// codes, key metadata, value codes, value metadata) of its next tile are
// copied into the warp's second slot with cp.async while it works on the
// current one, and the warp keeps its own online-softmax state.  The warps'
// states are merged once, in shared memory, after the last tile: no
// workspace, no CTA-wide barrier per tile.
//
// Per tile, the scores of the positions in pages are one tensor-core
// contraction per key group: with the key scale and zero constant over the
// group's kg positions of a channel,
//     q . k_t = sum_j (q_j scale_j) c_{t,j} + sum_j q_j zero_j,
// so q'_j = q_j scale_j (fp16 high and low parts, the query normalized per
// head by a power of two) forms the A rows (head, part) of m16n8k16 fp16
// products, the codes (exact in fp16) the B columns, channels the k
// dimension; the even and odd positions of a 16-position block are two
// n8 tiles, so that one byte of a channel run feeds both.  The second sum
// is a warp reduction per group.  Scores go to a per-warp table.  For the
// weighted values lane l owns channels 4l .. 4l+3 and walks the positions
// with the weights times value scale from a per-warp table, on CUDA cores:
// codes become floats by placing them in the mantissa of 1.0f
// (f = 1 + c 2^-bits, exact):
//     scale*c + zero = (scale 2^bits) f + (zero - scale 2^bits).
// Ring positions (at or above Q) are read as bf16 rows from global memory,
// prefetched into L2 when the tile's copies are issued; their scores are
// formed on CUDA cores by the lanes that own them (positions 2l, 2l+1).
#include <cuda_fp16.h>

#include "kvq_internal.cuh"
#include "kvq_tc_ptx.cuh"

namespace kvq {
namespace {

constexpr int PD = 128;
constexpr int PT = 64;              // positions per page (one tile)
constexpr int GMAX = 8;             // query heads per kv-head (kernels for up to 4 and up to 8)
// warps per CTA at most (about 200 registers per thread)
__host__ __device__ constexpr int nw_max(int nh) { return 8; }
constexpr int PHROW = 36;           // words per row of the fp16 weight table (32 used; the rest spreads banks)
constexpr int SMEM_MAX = 227 * 1024 - 256;   // dynamic bytes; the merge ticket is static
constexpr unsigned FULLM = 0xffffffffu;

// shared-memory geometry of one launch (bytes)
struct PcGeom {
    int KC, KM, VC, VM;     // the four raw blocks of a (page, kv-head)
    int SLOT;               // KC + KM + VC + VM
    int MT;                 // key (scale, zero) table: [PT/kg][PD] float2
    int PW;                 // weight table: [PT][nvg][NH] float
    int SS;                 // score table: [PT][NH] float
    int PH;                 // four heads: weight parts [nvg][8][36] fp16 pairs, zero sums [nvg][4]
    int WAREA;              // per warp: two slots, the tables
    int OFF_PAGES, OFF_AREAS;
    int NW, bytes;
};

__host__ __device__ inline int round_up(int x, int a) { return (x + a - 1) / a * a; }

constexpr int PSW = PD + 4;         // floats per (head) row of a part: PD outputs, maximum, weight sum, pad
// bytes of the split partials [pairs][splits][GMAX heads][PSW] (256-aligned)
inline size_t pc_part_bytes(int batch, int hkv, int splits) {
    return (size_t(batch) * hkv * splits * GMAX * PSW * 4 + 255) & ~size_t(255);
}

PcGeom pc_geometry(const Params& p, int max_len, int nh) {
    PcGeom g{};
    const int nkg = p.kg > 0 ? PT / p.kg : 1;
    g.KC = PD * PT * p.kb / 8;
    g.KM = nkg * PD * 4;
    g.VC = PD * PT * p.vb / 8;
    g.VM = PT * p.nvg * 4;
    g.SLOT = g.KC + g.KM + g.VC + g.VM;
    g.MT = nkg * PD * 8;
    g.PW = PT * p.nvg * nh * 4;
    g.SS = PT * nh * 4;
    g.PH = nh == 4 ? p.nvg * (8 * PHROW + 4) * 4 : 0;
    g.WAREA = round_up(2 * g.SLOT + g.MT + g.PW + g.SS + g.PH, 128);
    g.OFF_PAGES = PD * nh * 4 + 2 * nh * 4;
    g.OFF_AREAS = round_up(g.OFF_PAGES + 4 * (max_len / PT + 1), 128);
    const int nw = (SMEM_MAX - g.OFF_AREAS) / g.WAREA;
    g.NW = nw < nw_max(nh) ? nw : nw_max(nh);
    g.bytes = g.OFF_AREAS + (g.NW > 0 ? g.NW : 0) * g.WAREA;
    return g;
}

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
__device__ __forceinline__ void prefetch_l2(const void* a) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
}

// code c (BITS wide) found at bit `sh` of x, as the float 1 + c 2^-BITS: the
// code is moved to the top of the mantissa of 1.0f (shift, then one and-or)
template <int BITS>
__device__ __forceinline__ float code_f(uint32_t x, int sh) {
    constexpr int top = 23 - BITS;
    constexpr uint32_t mask = ((1u << BITS) - 1u) << top;
    const uint32_t y = sh <= top ? (x << (top - sh)) : (x >> (sh - top));
    return __uint_as_float((y & mask) | 0x3F800000u);
}
// the codes of positions 16 qt .. 16 qt + 15 of channel j's run (runs of
// BITS*8 bytes, chunk-major above 16 bytes: [chunk][d][min(16, run)]), as
// 16*BITS bits
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

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t h2bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
// both parts of the pair (x, y): the fp16 rounding, and the fp16 rounding of the rest
__device__ __forceinline__ void f16_parts(float x, float y, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(x, y);
    const float2 f = __half22float2(h);
    hi = h2bits(h);
    lo = h2bits(__floats2half2_rn(x - f.x, y - f.y));
}
// part `limb` (0: the fp16 rounding, 1: the fp16 rounding of the rest) of the pair (x, y)
__device__ __forceinline__ uint32_t f16_part(float x, float y, int limb) {
    const __half2 hi = __floats2half2_rn(x, y);
    const float2 f = __half22float2(hi);
    const __half2 lo = __floats2half2_rn(x - f.x, y - f.y);
    return limb ? h2bits(lo) : h2bits(hi);
}
// two codes (one per 16-bit half of y, BITS wide at bit 0) as an fp16 pair
template <int BITS>
__device__ __forceinline__ uint32_t codes_f16(uint32_t y) {
    constexpr uint32_t m = ((1u << BITS) - 1u) * 0x00010001u;
    const uint32_t biased = (y & m) | 0x64006400u;              // 1024 + c, exact
    const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&biased), __floats2half2_rn(1024.0f, 1024.0f));
    return h2bits(r);
}

// The weighted-value MMA's k slots (2 tig, 2 tig + 1) of register a0 hold the
// k-step's positions tig and tig + 8, those of a2 positions tig + 4 and
// tig + 12 (any order of k works when A and B agree; the weight table pairs
// the same positions).  A position p + 8 sits 8*BITS bits above p, so for
// 2-bit codes both halves come from one shift and one mask.  The codes of
// positions tig + 4 hf and tig + 4 hf + 8 of a k-step's words, as an fp16
// pair, the first in the low half.
template <int BITS, int HF>
__device__ __forceinline__ uint32_t vpair_f16(const uint32_t (&w)[4], int tig) {
    constexpr uint32_t m = (1u << BITS) - 1u;
    const int p = tig + 4 * HF;
    if constexpr (BITS == 1) {                      // bits p and p + 8 of the 16-bit word
        const uint32_t x = w[0] >> p;
        return codes_f16<1>((x & m) | ((x << 8) & (m << 16)));
    } else if constexpr (BITS == 2) {               // bits 2p and 2p + 16 of the word
        return codes_f16<2>(w[0] >> (2 * p));
    } else if constexpr (BITS == 4) {               // the same nibble of words 0 and 1
        return codes_f16<4>(__byte_perm(w[0] >> (4 * p), w[1] >> (4 * p), 0x5410));
    } else {                                        // byte p % 4 of word p / 4 and of word p / 4 + 2
        const uint32_t lo = (p >> 2) ? w[1] : w[0], hi = (p >> 2) ? w[3] : w[2];
        return codes_f16<8>(__byte_perm(lo, hi, uint32_t(p & 3) | (uint32_t((p & 3) + 4) << 8)));
    }
}
// the codes of positions 16 ks .. 16 ks + 15 of channel j's value run (2*BITS bytes)
template <int BITS>
__device__ __forceinline__ void vrun_kstep(const uint8_t* base, int j, int ks, uint32_t (&w)[4]) {
    constexpr int chan = PT * BITS / 8, cw = chan < 16 ? chan : 16;
    const int byte = 2 * BITS * ks;
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

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* a, unsigned v) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(a), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ float ld_relaxed_gpu(const float* a) {
    float v;
    asm volatile("ld.relaxed.gpu.f32 %0, [%1];" : "=f"(v) : "l"(a) : "memory");
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULLM, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULLM, v, o));
    return v;
}
__device__ __forceinline__ float ex2(float x) { return exp2f(x); }

template <int KB, int VB, int NH>
__global__ void __launch_bounds__(nw_max(NH) * 32, 1) decode_pc_kernel(const Params p, const void* __restrict__ qv,
                                                                  int q_bf16, const int32_t* __restrict__ lens,
                                                                  int max_len, float sl2, float* __restrict__ out,
                                                                  float* __restrict__ lse, const PcGeom geo,
                                                                  float* __restrict__ wpart, unsigned* tickets,
                                                                  const int S) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int h = blockIdx.x, b = blockIdx.y, split = blockIdx.z;   // split `split` of S of the pair's tiles
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, NW = blockDim.x >> 5;
    const int g = p.g, kg = p.kg, nvg = p.nvg;
    const int L = max(0, min(lens[b], max_len));
    const size_t orow0 = size_t(b) * p.hq + size_t(h) * g;
    if (L == 0) {                                   // an empty sequence: o = 0, lse = -inf (no split takes a ticket)
        if (split == 0)
        for (int e = tid; e < g * PD; e += blockDim.x) {
            out[(orow0 + e / PD) * PD + e % PD] = 0.0f;
            if (lse && e % PD == 0) lse[orow0 + e / PD] = -INFINITY;
        }
        return;
    }
    float* qf = reinterpret_cast<float*>(smem_raw);                          // [PD][NH], times sm_scale log2 e
    int* pages = reinterpret_cast<int*>(smem_raw + geo.OFF_PAGES);           // page ids of the quantized tiles
    uint8_t* areas = smem_raw + geo.OFF_AREAS;
    const int R = p.W + kg - 1;                     // ring slots
    const int Q = L - p.W > 0 ? ((L - p.W) / kg) * kg : 0;   // positions below Q live in pages
    const int ntiles_all = (L + PT - 1) / PT, npq = (Q + PT - 1) / PT;
    // this CTA's tiles [tile0, ntiles) of the pair's ntiles_all
    const int tile0 = int((long(ntiles_all) * split) / S), ntiles = int((long(ntiles_all) * (split + 1)) / S);
    const size_t prow = size_t(b) * p.hkv + h;      // (sequence, kv-head) row of the ring

    for (int e = tid; e < NH * PD; e += blockDim.x) {
        const int r = e / PD, j = e % PD;
        float x = 0.0f;
        if (r < g) {
            const size_t idx = (orow0 + r) * PD + j;
            x = q_bf16 ? bfbits(static_cast<const uint16_t*>(qv)[idx]) : static_cast<const float*>(qv)[idx];
        }
        qf[j * NH + r] = x * sl2;
    }
    for (int i = tid; i < npq; i += blockDim.x) {
        const int pg = i < p.max_pages ? p.page_table[size_t(b) * p.max_pages + i] : -1;
        pages[i] = pg >= p.num_pages ? -1 : pg;
    }
    __syncthreads();
    // per head a power of two that brings max_j |q_j| into [1/2, 1) (fp16 range
    // for q_j times a key scale), and its inverse
    float* hnorm = reinterpret_cast<float*>(smem_raw + PD * NH * 4);   // [NH] factor, [NH] inverse
    if (w == 0) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            float a = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) a = fmaxf(a, fabsf(qf[(4 * lane + c) * NH + r]));
            a = warp_max(a);
            const int eb = min(252, max(1, int(__float_as_uint(a) >> 23)));
            if (lane == 0) {
                hnorm[r] = a > 0.0f ? __uint_as_float(uint32_t(253 - eb) << 23) : 1.0f;      // 2^(126 - eb)
                hnorm[NH + r] = a > 0.0f ? __uint_as_float(uint32_t(eb + 1) << 23) : 1.0f;   // 2^(eb - 126)
            }
        }
    }
    __syncthreads();

    uint8_t* area = areas + size_t(w) * geo.WAREA;
    float2* mt = reinterpret_cast<float2*>(area + 2 * geo.SLOT);
    float* pw = reinterpret_cast<float*>(area + 2 * geo.SLOT + geo.MT);
    float* ss = reinterpret_cast<float*>(area + 2 * geo.SLOT + geo.MT + geo.PW);   // [PT][NH] scores
    uint32_t* ph = reinterpret_cast<uint32_t*>(area + 2 * geo.SLOT + geo.MT + geo.PW + geo.SS);
    float* crr = reinterpret_cast<float*>(ph + nvg * 8 * PHROW);                    // [nvg][4]
    // four heads: the weighted values of the positions in pages on tensor cores
    // (rows: channels, k: positions, columns: (head, part) of the weights)
    constexpr bool VMMA = NH == 4;
    const int lvg = __ffs(p.vg) - 1;                // value groups of 16 .. 128 channels
    const uint16_t* kwin = reinterpret_cast<const uint16_t*>(p.k_win) + prow * size_t(R) * PD;
    const uint16_t* vwin = reinterpret_cast<const uint16_t*>(p.v_win) + prow * size_t(R) * PD;

    // copies of tile i into slot s: the page's four blocks in 16-byte pieces
    // (zeros for an unmapped page); ring rows of the tile are prefetched to L2
    auto issue = [&](int i, int s) {
        if (i >= ntiles) return;
        const int t0 = i * PT;
        if (t0 < Q) {
            uint8_t* dst = area + s * geo.SLOT;
            const int pg = pages[i];
            if (pg < 0) {
                for (int c = lane; c < geo.SLOT / 16; c += 32)
                    *reinterpret_cast<uint4*>(dst + 16 * c) = make_uint4(0u, 0u, 0u, 0u);
            } else {
                const size_t blk = size_t(pg) * p.hkv + h;
                const uint32_t d0 = ptx::smem_u32(dst);
                const uint8_t* kc = p.k_codes + blk * geo.KC;
                const uint8_t* km = reinterpret_cast<const uint8_t*>(p.k_meta) + blk * geo.KM;
                const uint8_t* vc = p.v_codes + blk * geo.VC;
                const uint8_t* vm = reinterpret_cast<const uint8_t*>(p.v_meta) + blk * geo.VM;
                for (int c = lane; c < geo.KC / 16; c += 32) cpa16(d0 + 16 * c, kc + 16 * c);
                for (int c = lane; c < geo.KM / 16; c += 32) cpa16(d0 + geo.KC + 16 * c, km + 16 * c);
                for (int c = lane; c < geo.VC / 16; c += 32) cpa16(d0 + geo.KC + geo.KM + 16 * c, vc + 16 * c);
                for (int c = lane; c < geo.VM / 16; c += 32)
                    cpa16(d0 + geo.KC + geo.KM + geo.VC + 16 * c, vm + 16 * c);
            }
        }
        // ring positions of the tile: 256-byte key and value rows, two lines each
        const int w0 = max(t0, Q), w1 = min(t0 + PT, L);
        for (int e = lane; e < 4 * (w1 - w0); e += 32) {
            const int t = w0 + (e >> 2), part = e & 3;
            const uint16_t* row = ((part & 2) ? vwin : kwin) + size_t(t % R) * PD + (part & 1) * 64;
            prefetch_l2(row);
        }
    };

    float m_run[NH], l_run[NH], o[NH][4];
#pragma unroll
    for (int r = 0; r < NH; ++r) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.0f;
        o[r][0] = o[r][1] = o[r][2] = o[r][3] = 0.0f;
    }
    // four heads: channels 16 mt + g8 (+ 8) of head tig, high and low weight parts
    float ov[VMMA ? 8 : 1][4];
#pragma unroll
    for (int mt = 0; mt < (VMMA ? 8 : 1); ++mt) ov[mt][0] = ov[mt][1] = ov[mt][2] = ov[mt][3] = 0.0f;
    // positions of this lane in the tile (scores, softmax, weight table): p and
    // p + 8 of the lane's 16-position block, the pairs the value MMA's k slots take
    const int tA = 16 * (lane >> 3) + (lane & 7), tB = tA + 8;
    const int j0 = 4 * lane;                        // value channels of this lane
    const int gv = j0 / p.vg;                       // their value group

    constexpr int kchan = PT * KB / 8, kcw = kchan < 16 ? kchan : 16;   // key run, chunk bytes
    const int g8 = lane >> 2, tig = lane & 3;       // fragment row group, thread in group
    const int r0 = g8 >> 1, limb = g8 & 1;          // A row g8: head r0, part limb (row g8 + 8: head r0 + 4)
    float f0 = 1.0f, f1 = 1.0f, i0 = 1.0f, i1 = 1.0f;   // normalization of heads r0 (and r0 + 4)
#pragma unroll
    for (int r = 0; r < NH; ++r) {
        if (r == r0) f0 = hnorm[r], i0 = hnorm[NH + r];
        if (NH == 8 && r == r0 + 4) f1 = hnorm[r], i1 = hnorm[NH + r];
    }

    int slot = 0;
    issue(tile0 + w, 0);
    cpa_commit();
    for (int i = tile0 + w; i < ntiles; i += NW) {
        issue(i + NW, slot ^ 1);
        cpa_commit();
        cpa_wait_1();
        __syncwarp();                               // every lane's pieces of tile i have landed
        const int t0 = i * PT;
        const int nq = min(PT, max(0, Q - t0));     // quantized positions of the tile (a multiple of kg)
        const int nv = min(PT, L - t0);             // valid positions of the tile
        const uint8_t* raw = area + slot * geo.SLOT;
        const uint8_t* kc = raw;
        const uint32_t* km = reinterpret_cast<const uint32_t*>(raw + geo.KC);
        const uint8_t* vc = raw + geo.KC + geo.KM;
        const uint32_t* vm = reinterpret_cast<const uint32_t*>(raw + geo.KC + geo.KM + geo.VC);

        // ---- key groups of the tile: (scale, zero) per channel
        if (nq > 0) {
            for (int e = lane; e < (nq / kg) * PD; e += 32) {
                const uint32_t m = km[e];
                mt[e] = make_float2(hbits(m & 0xffffu), hbits(m >> 16));
            }
        }
        __syncwarp();

        // ---- scores of the positions in the page, per key group (tensor cores)
        for (int gi = 0; gi < nq / kg; ++gi) {
            const float2* mg = mt + gi * PD;
            // the zero-point sum of every head: channels 4l .. 4l+3, then the warp
            float bz[NH];
#pragma unroll
            for (int r = 0; r < NH; ++r) bz[r] = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float z = mg[4 * lane + c].y;
                float qq[NH];
                ld_heads<NH>(qf + (4 * lane + c) * NH, qq);
#pragma unroll
                for (int r = 0; r < NH; ++r) bz[r] = fmaf(qq[r], z, bz[r]);
            }
            float b0 = 0.0f, b1 = 0.0f;
#pragma unroll
            for (int r = 0; r < NH; ++r) {
                const float t = warp_sum(bz[r]);
                if (r == r0) b0 = t;
                if (NH == 8 && r == r0 + 4) b1 = t;
            }
            // A fragments: rows (head, part) of q_j 2^-e scale_j, channels 16 ks + {2tig, +1, +8, +9}
            uint32_t af[8][4];
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int c = 16 * ks + 2 * tig + 8 * hf;
                    const float s0 = mg[c].x, s1 = mg[c + 1].x;
                    af[ks][2 * hf] = f16_part(qf[c * NH + r0] * f0 * s0, qf[(c + 1) * NH + r0] * f0 * s1, limb);
                    af[ks][2 * hf + 1] =
                        NH == 8 ? f16_part(qf[c * NH + r0 + 4] * f1 * s0, qf[(c + 1) * NH + r0 + 4] * f1 * s1, limb)
                                : 0u;
                }
            }
            // 16-position blocks of the group: even and odd positions as two n8 tiles
            for (int blk = gi * (kg / 16); blk < (gi + 1) * (kg / 16); ++blk) {
                const int bit = (16 * blk + 2 * g8) * KB, byte = bit >> 3, sh = bit & 7;
                const uint8_t* kb0 = kc + (byte / kcw) * (PD * kcw) + (byte % kcw);
                float de[4] = {0.0f, 0.0f, 0.0f, 0.0f}, dd[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int c0 = 16 * ks + 2 * tig;
                    uint32_t x[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c = c0 + (u & 1) + 8 * (u >> 1);
                        if constexpr (KB == 8) x[u] = *reinterpret_cast<const uint16_t*>(kb0 + c * kcw);
                        else x[u] = kb0[c * kcw];
                    }
                    const uint32_t y01 = __byte_perm(x[0], x[1], 0x5410) >> sh;
                    const uint32_t y23 = __byte_perm(x[2], x[3], 0x5410) >> sh;
                    const uint32_t a4[4] = {af[ks][0], af[ks][1], af[ks][2], af[ks][3]};
                    mma_f16(de, a4, codes_f16<KB>(y01), codes_f16<KB>(y23));
                    mma_f16(dd, a4, codes_f16<KB>(y01 >> KB), codes_f16<KB>(y23 >> KB));
                }
                // rows g8 and g8 ^ 1 are the two parts of one head: lanes 4 apart
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    de[i] += __shfl_xor_sync(FULLM, de[i], 4);
                    dd[i] += __shfl_xor_sync(FULLM, dd[i], 4);
                }
                // lane (g8, tig) holds positions 16 blk + 4 tig + {0 (de), 1 (dd), 2 (de), 3 (dd)};
                // the lanes of part 0 store the even ones, those of part 1 the odd ones
                const float* d = limb ? dd : de;
                const int t0p = 16 * blk + 4 * tig + limb;
                ss[t0p * NH + r0] = fmaf(d[0], i0, b0);
                ss[(t0p + 2) * NH + r0] = fmaf(d[1], i0, b0);
                if (NH == 8) {
                    ss[t0p * NH + r0 + 4] = fmaf(d[2], i1, b1);
                    ss[(t0p + 2) * NH + r0 + 4] = fmaf(d[3], i1, b1);
                }
            }
        }
        __syncwarp();

        // ---- scores of positions tA, tB for every head (log2 domain)
        float sA[NH], sB[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r) sA[r] = sB[r] = 0.0f;
        if (tA < nq) {
            ld_heads<NH>(ss + tA * NH, sA);
            ld_heads<NH>(ss + tB * NH, sB);
        } else if (tA < nv) {
            const bool hasB = tB < nv;
            const uint16_t* ra = kwin + size_t((t0 + tA) % R) * PD;
            const uint16_t* rb = hasB ? kwin + size_t((t0 + tB) % R) * PD : ra;
#pragma unroll 2
            for (int j8 = 0; j8 < PD; j8 += 8) {
                const uint4 a = *reinterpret_cast<const uint4*>(ra + j8);
                const uint4 c = *reinterpret_cast<const uint4*>(rb + j8);
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float kA = bfbits((aw[e >> 1] >> (16 * (e & 1))) & 0xffffu);
                    const float kB = bfbits((cw[e >> 1] >> (16 * (e & 1))) & 0xffffu);
                    float qq[NH];
                    ld_heads<NH>(qf + (j8 + e) * NH, qq);
#pragma unroll
                    for (int r = 0; r < NH; ++r) {
                        sA[r] = fmaf(qq[r], kA, sA[r]);
                        sB[r] = fmaf(qq[r], kB, sB[r]);
                    }
                }
            }
        }
        const bool vA = tA < nv, vB = tB < nv;

        // ---- online softmax over the tile, per head
        float pA[NH], pB[NH], alpha[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r) {
            const float mx = warp_max(fmaxf(vA ? sA[r] : -INFINITY, vB ? sB[r] : -INFINITY));
            const float mn = fmaxf(m_run[r], mx);    // finite: position t0 < L is in the tile
            alpha[r] = ex2(m_run[r] - mn);           // 0 on the warp's first tile
            m_run[r] = mn;
            pA[r] = vA ? ex2(sA[r] - mn) : 0.0f;
            pB[r] = vB ? ex2(sB[r] - mn) : 0.0f;
            l_run[r] = fmaf(l_run[r], alpha[r], warp_sum(pA[r] + pB[r]));
#pragma unroll
            for (int c = 0; c < 4; ++c) o[r][c] *= alpha[r];
        }
        if constexpr (VMMA) {
            float at = alpha[0];
#pragma unroll
            for (int r = 1; r < NH; ++r) at = tig == r ? alpha[r] : at;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) ov[mt][i] *= at;
        }

        // ---- weight tables.  Eight heads: [t][value group][head] on CUDA cores,
        // positions in pages p*scale*2^VB, ring positions p; per value group the
        // zero points and the mantissa offsets: sum_t p (zero - scale 2^VB).
        // Four heads: positions in pages as fp16 parts of p*scale, [group][(head,
        // part)][word] (lane l writes word l: its positions tA, tB), and the zero
        // sums sum_t p zero per group; ring positions p in the float table.
        float corr[NH];
#pragma unroll
        for (int r = 0; r < NH; ++r) corr[r] = 0.0f;
        for (int gg = 0; gg < nvg; ++gg) {
            float z[NH];
#pragma unroll
            for (int r = 0; r < NH; ++r) z[r] = 0.0f;
            if (VMMA && tA < nq) {
                const uint32_t mA = vm[tA * nvg + gg], mB = vm[tB * nvg + gg];
                const float sa = hbits(mA & 0xffffu), sb = hbits(mB & 0xffffu);
                const float za = hbits(mA >> 16), zb = hbits(mB >> 16);
#pragma unroll
                for (int r = 0; r < NH; ++r) {
                    uint32_t hi, lo;
                    f16_parts(pA[r] * sa, pB[r] * sb, hi, lo);
                    ph[(gg * 8 + 2 * r) * PHROW + lane] = hi;
                    ph[(gg * 8 + 2 * r + 1) * PHROW + lane] = lo;
                    z[r] = fmaf(pA[r], za, fmaf(pB[r], zb, z[r]));
                }
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int t = half ? tB : tA;
                const float* pp = half ? pB : pA;
                if (t >= nv || (VMMA && t < nq)) continue;
                float wt[NH];
                if (t < nq) {
                    const uint32_t m = vm[t * nvg + gg];
                    const float s = hbits(m & 0xffffu) * float(1 << VB), zz = hbits(m >> 16) - s;
#pragma unroll
                    for (int r = 0; r < NH; ++r) {
                        wt[r] = pp[r] * s;
                        z[r] = fmaf(pp[r], zz, z[r]);
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < NH; ++r) wt[r] = pp[r];
                }
#pragma unroll
                for (int r = 0; r < NH; r += 4)
                    *reinterpret_cast<float4*>(pw + (t * nvg + gg) * NH + r) =
                        make_float4(wt[r], wt[r + 1], wt[r + 2], wt[r + 3]);
            }
            if (nq > 0) {
#pragma unroll
                for (int r = 0; r < NH; ++r) {
                    const float zs = warp_sum(z[r]);
                    if (gg == gv) corr[r] = zs;
                    if (VMMA && lane == 0) crr[gg * 4 + r] = zs;
                }
            }
        }
        __syncwarp();                               // the weight tables are complete

        if constexpr (VMMA) {
            // ---- o += sum_t w_t v_t, positions in pages: 8 channel tiles x nq/16 k-steps
            for (int ks = 0; ks < nq / 16; ++ks) {
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    const int ja = 16 * mt + g8, gvm = (16 * mt) >> lvg;
                    uint32_t wa[4], wb[4];
                    vrun_kstep<VB>(vc, ja, ks, wa);
                    vrun_kstep<VB>(vc, ja + 8, ks, wb);
                    const uint32_t a4[4] = {vpair_f16<VB, 0>(wa, tig), vpair_f16<VB, 0>(wb, tig),
                                            vpair_f16<VB, 1>(wa, tig), vpair_f16<VB, 1>(wb, tig)};
                    const uint32_t* prow = ph + (gvm * 8 + g8) * PHROW + 8 * ks + tig;
                    mma_f16(ov[mt], a4, prow[0], prow[4]);
                }
            }
            if (nq > 0) {
                // zero points of the positions in pages, once per (channel, head) in the high part
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    const float zc = crr[((16 * mt) >> lvg) * 4 + tig];
                    ov[mt][0] += zc;
                    ov[mt][2] += zc;
                }
            }
        } else {
            // ---- o += sum_t w_t v_t over the tile: channels j0 .. j0+3
            for (int qt = 0; qt < nq / 16; ++qt) {
                uint32_t cw4[4][4];
#pragma unroll
                for (int c = 0; c < 4; ++c) run_quarter<VB>(vc, j0 + c, qt, cw4[c]);
#pragma unroll
                for (int tt = 0; tt < 16; ++tt) {
                    float pq[NH];
                    ld_heads<NH>(pw + ((16 * qt + tt) * nvg + gv) * NH, pq);
                    const int bit = tt * VB;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float f = code_f<VB>(cw4[c][bit >> 5], bit & 31);
#pragma unroll
                        for (int r = 0; r < NH; ++r) o[r][c] = fmaf(pq[r], f, o[r][c]);
                    }
                }
            }
        }
#pragma unroll 4
        for (int t = nq; t < nv; ++t) {
            const uint2 v = *reinterpret_cast<const uint2*>(vwin + size_t((t0 + t) % R) * PD + j0);
            const float x[4] = {bfbits(v.x & 0xffffu), bfbits(v.x >> 16), bfbits(v.y & 0xffffu), bfbits(v.y >> 16)};
            float pq[NH];
            ld_heads<NH>(pw + (t * nvg + gv) * NH, pq);
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int r = 0; r < NH; ++r) o[r][c] = fmaf(pq[r], x[c], o[r][c]);
        }
        if constexpr (!VMMA) {
#pragma unroll
            for (int r = 0; r < NH; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) o[r][c] += corr[r];
        }
        __syncwarp();                               // slot, tables free for the next tiles
        slot ^= 1;
    }
    cpa_wait_0();
    __syncthreads();                                // every warp is done with its area

    // ---- merge the warps' states: [warp][head][PD + 2] over the warp areas
    constexpr int PS = PD + 4;
    float* part = reinterpret_cast<float*>(areas);
#pragma unroll
    for (int r = 0; r < NH; ++r) {
        if (r >= g) break;
        *reinterpret_cast<float4*>(part + (w * NH + r) * PS + j0) = make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
        if (lane == 0) {
            part[(w * NH + r) * PS + PD] = m_run[r];
            part[(w * NH + r) * PS + PD + 1] = l_run[r];
        }
    }
    if constexpr (VMMA) {
        __syncwarp();                               // the CUDA-core part of the warp's rows first
        if (tig < g) {
            float* prt = part + (w * NH + tig) * PS;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                prt[16 * mt + g8] += ov[mt][0] + ov[mt][1];
                prt[16 * mt + g8 + 8] += ov[mt][2] + ov[mt][3];
            }
        }
    }
    __syncthreads();
    // a pair split between CTAs: this CTA's merged part goes to the workspace,
    // [pair][split][head][PS]: the unnormalized output, the maximum (log2
    // domain) and the weight sum
    const size_t pair = size_t(b) * p.hkv + h;
    float* wp = S > 1 ? wpart + (pair * S + split) * size_t(GMAX * PS) : nullptr;
    for (int e = tid; e < g * PD; e += blockDim.x) {
        const int r = e / PD, j = e % PD;
        float M = -INFINITY;
        for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, part[(ww * NH + r) * PS + PD]);
        float num = 0.0f, den = 0.0f;
        for (int ww = 0; ww < NW; ++ww) {
            const float mw = part[(ww * NH + r) * PS + PD];
            if (mw == -INFINITY) continue;          // a warp without tiles
            const float f = ex2(mw - M);
            num = fmaf(part[(ww * NH + r) * PS + j], f, num);
            den = fmaf(part[(ww * NH + r) * PS + PD + 1], f, den);
        }
        if (S == 1) {
            out[(orow0 + r) * PD + j] = num / den;
            if (lse && j == 0) lse[orow0 + r] = (M + log2f(den)) * 0.693147180559945309f;
        } else {
            wp[r * PS + j] = num;
            if (j == 0) {
                wp[r * PS + PD] = M;
                wp[r * PS + PD + 1] = den;
            }
        }
    }
    if (S == 1) return;
    // every thread's part, then the ticket (release); the CTA that takes the
    // pair's last ticket (acquire) merges every split's part in split order,
    // so that the result does not depend on which CTA finished last, and
    // resets the ticket for the next call.  No CTA waits for another.
    __shared__ unsigned ticket;
    __syncthreads();
    if (tid == 0) ticket = atom_add_acq_rel_gpu(tickets + pair, 1u);
    __syncthreads();
    if (ticket != unsigned(S - 1)) return;
    const float* wq = wpart + pair * S * size_t(GMAX * PS);
    for (int e = tid; e < g * PD; e += blockDim.x) {
        const int r = e / PD, j = e % PD;
        float M = -INFINITY;
        for (int sp = 0; sp < S; ++sp) M = fmaxf(M, ld_relaxed_gpu(wq + (size_t(sp) * GMAX + r) * PS + PD));
        float num = 0.0f, den = 0.0f;
        for (int sp = 0; sp < S; ++sp) {
            const float* q2 = wq + (size_t(sp) * GMAX + r) * PS;
            const float ms = ld_relaxed_gpu(q2 + PD);
            if (ms == -INFINITY) continue;          // a split without positions
            const float f = ex2(ms - M);
            num = fmaf(ld_relaxed_gpu(q2 + j), f, num);
            den = fmaf(ld_relaxed_gpu(q2 + PD + 1), f, den);
        }
        out[(orow0 + r) * PD + j] = num / den;
        if (lse && j == 0) lse[orow0 + r] = (M + log2f(den)) * 0.693147180559945309f;
    }
    if (tid == 0) tickets[pair] = 0u;               // ready for the next call
}

template <int KB, int NH>
cudaError_t launch_nh_pc(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len, float sl2,
                         float* out, float* lse, void* ws, int S, cudaStream_t s) {
    const PcGeom geo = pc_geometry(p, max_len, NH);
    const dim3 grid(p.hkv, p.batch, S);
    float* wpart = S > 1 ? static_cast<float*>(ws) : nullptr;
    unsigned* tickets = S > 1 ? reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) + pc_part_bytes(p.batch, p.hkv, S))
                              : nullptr;
    auto go = [&](auto kern) -> cudaError_t {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, geo.bytes);
        if (e != cudaSuccess) return e;
        kern<<<grid, geo.NW * 32, geo.bytes, s>>>(p, q, q_bf16, lens, max_len, sl2, out, lse, geo, wpart, tickets, S);
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
                         float* out, float* lse, void* ws, int S, cudaStream_t s) {
    if (p.g <= 4) return launch_nh_pc<KB, 4>(p, q, q_bf16, lens, max_len, sl2, out, lse, ws, S, s);
    return launch_nh_pc<KB, 8>(p, q, q_bf16, lens, max_len, sl2, out, lse, ws, S, s);
}

}  // namespace

bool decode_pc_supported(const Params& p, int max_len) {
    if (!(p.d == PD && p.g >= 1 && p.g <= GMAX && (p.kg == 16 || p.kg == 32 || p.kg == 64) && p.vg >= 16 &&
          PD % p.vg == 0 && !p.rotate && max_len >= 0))
        return false;
    // two warps at least, each with two page slots and its tables
    return pc_geometry(p, max_len, p.g <= 4 ? 4 : 8).NW >= 2;
}

int pc_splits(const Params& p, int batch, int max_len, int sms) {
    const long pairs = long(batch) * p.hkv;
    if (pairs <= 0) return 1;
    long S = sms / pairs;                           // every CTA in one wave (one CTA per SM)
    const long by_len = (long(max_len) + PT - 1) / PT / nw_max(8);   // eight tiles per CTA at least
    if (S > by_len) S = by_len;
    if (S > 8) S = 8;
    return S < 1 ? 1 : int(S);
}

size_t pc_workspace_bytes(const Params& p, int batch, int splits) {
    return pc_part_bytes(batch, p.hkv, splits) + size_t(batch) * p.hkv * 4;
}

cudaError_t launch_decode_per_channel(const Params& p, const void* q, int q_bf16, const int32_t* lens, int max_len,
                                      float sm_scale, float* out, float* lse, void* ws, int splits, cudaStream_t s) {
    const float sl2 = sm_scale * 1.4426950408889634f;
    const int S = splits > 1 && ws ? splits : 1;
    switch (p.kb) {
        case 1: return launch_kb_pc<1>(p, q, q_bf16, lens, max_len, sl2, out, lse, ws, S, s);
        case 2: return launch_kb_pc<2>(p, q, q_bf16, lens, max_len, sl2, out, lse, ws, S, s);
        case 4: return launch_kb_pc<4>(p, q, q_bf16, lens, max_len, sl2, out, lse, ws, S, s);
        default: return launch_kb_pc<8>(p, q, q_bf16, lens, max_len, sl2, out, lse, ws, S, s);
    }
}

}  // namespace kvq

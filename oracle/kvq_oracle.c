/*
 * kvq_oracle.c -- plain, slow, CPU oracle for the mixed-precision quantized
 * KV cache (group-wise asymmetric low-bit codes, more bits for keys than for
 * values) and for single-token decode attention over it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Sources (web pages; quoted by title and section):
 *  [P1] "Kuantisasi KV cache mengganggu attention melalui key dan value
 *       tersimpan" (nalar.dev): sections "Error pada key masuk sebelum
 *       softmax" (s = qK^T/sqrt(d), a = softmax(s), o = aV), "Error pada
 *       value masuk setelah bobot attention terbentuk", "Granularitas
 *       kuantisasi menentukan nilai yang berbagi scale" (a group of values
 *       shares one scale and a zero point / offset), "Pertumbuhan cache
 *       mengubah trade pada serving" (recent tokens kept at higher precision,
 *       older blocks quantized).
 *  [P2] "Kuantisasi on Nalar" tag index: teaser "Kuantisasi KV Cache
 *       Mengurangi State Attention dengan Biaya Rekonstruksi" (entries are
 *       encoded with fewer bits plus scale / zero-point metadata and
 *       reconstructed when attention uses them).
 *  [P3] "Quantize What Counts: More for Keys, Less for Values" (technical
 *       summary of arXiv 2502.15075): Methodologie / Belangrijkste Bijdragen
 *       (K4V2, key-driven bit allocation), Resultaten (key groups of 32,
 *       value groups of 64 or 128; rotation applied to keys only).
 *
 * The pages print no quantizer formula.  This oracle takes the plainest
 * reading: per group, fp32 min/max; zero point = fp16(min) rounded down;
 * scale = fp16((max - zero) / (2^b - 1)) with every step rounded up, so the
 * code grid [zero, zero + (2^b-1)*scale] covers the group; code =
 * rint((x - zero) / scale) clamped to [0, 2^b - 1]; reconstruction
 * x^ = code * scale + zero (one fused multiply-add in fp32).  Attention is
 * evaluated in fp64 on the reconstructed values.
 *
 * Build: gcc -O2 -fPIC -shared -frounding-math -ffp-contract=off -fopenmp
 * (no fast-math: every fp32 step below is one IEEE-754 operation).
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KVQO_OK 0
#define KVQO_ERR_ARG (-1)
#define KVQO_ERR_UNSUPPORTED (-2)

/* rounding directions for the format conversion below */
#define KVQO_RN 0   /* to nearest, ties to even */
#define KVQO_RD (-1) /* toward -infinity */
#define KVQO_RU 1   /* toward +infinity */

/* ------------------------------------------------------------------------
 * Rounding a real (held exactly in a double) into a binary floating-point
 * format with p significand bits (implicit bit included), minimum normal
 * exponent emin and largest finite value maxf.  Written from the IEEE 754
 * definition of the formats: in the binade [2^e, 2^(e+1)) the representable
 * numbers are the multiples of 2^(e-p+1); below 2^emin they are the
 * multiples of 2^(emin-p+1) (subnormals).  The result is the grid point
 * chosen by the rounding direction; above the largest finite value the
 * result is infinity, except when a directed mode rounds the magnitude
 * down, which gives maxf.
 * ---------------------------------------------------------------------- */
static double round_to_format(double x, int p, int emin, double maxf, int mode)
{
    if (x == 0.0 || isinf(x)) return x;
    int neg = x < 0;
    double a = fabs(x);
    int e;
    frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                /* now 2^e <= a < 2^(e+1) */
    int qexp = (e < emin ? emin : e) - (p - 1);  /* exponent of one ulp */
    double m = ldexp(a, -qexp);                  /* exact: power-of-2 scaling */
    double lo = floor(m), hi = ceil(m), k;
    if (lo == m) {
        k = m;
    } else {
        int up;
        if (mode == KVQO_RN) {
            double frac = m - lo;
            up = frac > 0.5 || (frac == 0.5 && fmod(lo, 2.0) != 0.0);
        } else if (mode == KVQO_RU) {
            up = !neg;     /* toward +inf: magnitude grows for positives */
        } else {
            up = neg;      /* toward -inf: magnitude grows for negatives */
        }
        k = up ? hi : lo;
    }
    double v = ldexp(k, qexp);
    if (v > maxf) {
        int mag_down = (mode == KVQO_RU && neg) || (mode == KVQO_RD && !neg);
        v = mag_down ? maxf : INFINITY;
    }
    return neg ? -v : v;
}

/* binary16: p = 11, emin = -14, max 65504; bits = sign | exp(5) | frac(10) */
uint16_t kvqo_f32_to_f16(float x, int mode)
{
    if (isnan(x)) return (uint16_t)(signbit(x) ? 0xFE00u : 0x7E00u);   /* NaN stays NaN (quiet) */
    double v = round_to_format((double)x, 11, -14, 65504.0, mode);
    uint16_t s = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a == 0.0) return s;
    if (isinf(a)) return (uint16_t)(s | 0x7C00u);
    if (a < ldexp(1.0, -14)) {                      /* subnormal */
        return (uint16_t)(s | (uint16_t)ldexp(a, 24));
    }
    int e;
    frexp(a, &e);
    e -= 1;
    uint32_t frac = (uint32_t)(ldexp(a, 10 - e) - 1024.0);
    return (uint16_t)(s | (uint16_t)((e + 15) << 10) | frac);
}

float kvqo_f16_to_f32(uint16_t h)
{
    int s = h >> 15, ex = (h >> 10) & 31, fr = h & 1023;
    double v;
    if (ex == 0) v = ldexp((double)fr, -24);
    else if (ex == 31) v = fr ? NAN : INFINITY;
    else v = ldexp((double)(fr + 1024), ex - 25);
    return (float)(s ? -v : v);
}

/* bfloat16: p = 8, emin = -126, max (2 - 2^-7) * 2^127 */
uint16_t kvqo_f32_to_bf16(float x, int mode)
{
    double maxf = ldexp(255.0, 120);
    double v = round_to_format((double)x, 8, -126, maxf, mode);
    float f = (float)v;                   /* exact: v is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

float kvqo_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------------
 * Single IEEE-754 fp32 operations in a chosen rounding direction.  The
 * volatile accesses keep each operation between the two mode switches.
 * ---------------------------------------------------------------------- */
static float op_mode(float a, float b, int op, int rmode)
{
    volatile float va = a, vb = b, r;
    int old = fegetround();
    fesetround(rmode);
    if (op == 0) r = va - vb;
    else r = va / vb;
    fesetround(old);
    return r;
}
float kvqo_sub_ru(float a, float b) { return op_mode(a, b, 0, FE_UPWARD); }
float kvqo_div_ru(float a, float b) { return op_mode(a, b, 1, FE_UPWARD); }
/* Round-to-nearest is the default mode of the process (the oracle never
 * leaves another mode set), so these are the plain IEEE operations. */
float kvqo_sub_rn(float a, float b) { volatile float va = a, vb = b; return va - vb; }
float kvqo_div_rn(float a, float b) { volatile float va = a, vb = b; return va / vb; }

/* ------------------------------------------------------------------------
 * Group quantizer.  [P1] "Granularitas kuantisasi ...": a group of values
 * is mapped through one scale and a zero point; [P2] "... Biaya
 * Rekonstruksi": the metadata is scale and zero point.  Formula as stated
 * in the file header.
 * ---------------------------------------------------------------------- */
void kvqo_quantize_group(const float* x, int n, int bits,
                         uint16_t* scale_h, uint16_t* zero_h, uint8_t* codes)
{
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
    }
    if (mn == 0.0f) mn = 0.0f;   /* -0 and +0 compare equal: store +0 */
    if (mx == 0.0f) mx = 0.0f;
    const float qmax = (float)((1 << bits) - 1);
    uint16_t zh = kvqo_f32_to_f16(mn, KVQO_RD);
    float zf = kvqo_f16_to_f32(zh);
    float r = kvqo_sub_ru(mx, zf);
    float s32 = kvqo_div_ru(r, qmax);
    uint16_t sh = kvqo_f32_to_f16(s32, KVQO_RU);
    float sf = kvqo_f16_to_f32(sh);
    if (sf == 0.0f) sh = 0;
    *scale_h = sh;
    *zero_h = zh;
    for (int i = 0; i < n; ++i) {
        if (sf == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float t = kvqo_div_rn(kvqo_sub_rn(x[i], zf), sf);
        float c = nearbyintf(t);            /* default mode: ties to even */
        if (c < 0.0f) c = 0.0f;
        if (c > qmax) c = qmax;
        codes[i] = (uint8_t)c;
    }
}

/* reconstruction x^ = code * scale + zero, one fp32 fused multiply-add */
float kvqo_dequant_code(uint8_t code, uint16_t scale_h, uint16_t zero_h)
{
    return fmaf((float)code, kvqo_f16_to_f32(scale_h), kvqo_f16_to_f32(zero_h));
}

/* ------------------------------------------------------------------------
 * Bit packing (this library's storage format).  Little-endian: element i of
 * a packed run of b-bit codes sits in bits [b*(i mod (32/b)), +b) of 32-bit
 * word floor(i*b/32); words are stored little-endian.
 * ---------------------------------------------------------------------- */
void kvqo_pack(const uint8_t* codes, int n, int bits, uint8_t* out)
{
    int per = 32 / bits;
    int nwords = (n * bits + 31) / 32;
    for (int w = 0; w < nwords; ++w) {
        uint32_t word = 0;
        for (int i = 0; i < per && w * per + i < n; ++i)
            word |= (uint32_t)codes[w * per + i] << (bits * i);
        out[4 * w + 0] = (uint8_t)(word);
        out[4 * w + 1] = (uint8_t)(word >> 8);
        out[4 * w + 2] = (uint8_t)(word >> 16);
        out[4 * w + 3] = (uint8_t)(word >> 24);
    }
}

uint8_t kvqo_unpack_one(const uint8_t* packed, int i, int bits)
{
    int per = 32 / bits;
    const uint8_t* p = packed + 4 * (i / per);
    uint32_t word = (uint32_t)p[0] | ((uint32_t)p[1] << 8) |
                    ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
    return (uint8_t)((word >> (bits * (i % per))) & ((1u << bits) - 1u));
}

static void set_packed(uint8_t* packed, int i, int bits, uint8_t code)
{
    int per = 32 / bits;
    uint8_t* p = packed + 4 * (i / per);
    uint32_t word = (uint32_t)p[0] | ((uint32_t)p[1] << 8) |
                    ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
    uint32_t mask = ((1u << bits) - 1u) << (bits * (i % per));
    word = (word & ~mask) | (((uint32_t)code << (bits * (i % per))) & mask);
    p[0] = (uint8_t)word;
    p[1] = (uint8_t)(word >> 8);
    p[2] = (uint8_t)(word >> 16);
    p[3] = (uint8_t)(word >> 24);
}

/* ------------------------------------------------------------------------
 * Walsh-Hadamard rotation of keys ([P3] Resultaten, "Rotatie-integratie":
 * rotation applied to keys only).  H is the Sylvester-ordered Hadamard
 * matrix H[i][j] = (-1)^popcount(i & j); the rotation is
 * y = (x * sigma) H / sqrt(d) with sigma a +-1 diagonal, evaluated as a
 * dense product in fp64 and rounded once to fp32.
 * ---------------------------------------------------------------------- */
void kvqo_hadamard(int n, double* H)
{
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j)
            H[i * n + j] = (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0;
}

void kvqo_rotate_f64(const double* x, const int8_t* signs, int d, double* y)
{
    double inv = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) {
            double h = (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0;
            acc += h * ((double)signs[j] * x[j]);
        }
        y[i] = acc * inv;
    }
}

void kvqo_rotate(const float* x, const int8_t* signs, int d, float* y)
{
    double xd[256] = {0}, yd[256];
    if (d <= 0 || d > 256) return;      /* head_dim is at most 256 (check_layout) */
    for (int j = 0; j < d; ++j) xd[j] = x[j];
    kvqo_rotate_f64(xd, signs, d, yd);
    for (int i = 0; i < d; ++i) y[i] = (float)yd[i];
}

/* ------------------------------------------------------------------------
 * Cache layout (this library's storage format; the oracle writes it out on
 * its own).  Per layer:
 *   k_codes [pages][Hkv][P][d*kb/8]       token rows, channels packed
 *           (rows over 16 bytes stored as 16-byte chunks, chunk-major)
 *   k_meta  [pages][Hkv][P][d/kg] {u16 scale, u16 zero}
 *   v_codes [pages][Hkv][d][P*vb/8]       channel rows, tokens packed
 *           (likewise chunk-major when over 16 bytes)
 *   v_meta  [pages][Hkv][P][d/vg] {u16 scale, u16 zero}
 *   k_win, v_win [B][Hkv][W][d] bf16 ring, slot = position mod W
 *   page_table [B][max_pages] int32
 * Positions [0, L-W) live in pages (position p in logical page p/P, slot
 * p%P); the last min(W, L) positions live in the ring ([P1] "Pertumbuhan
 * cache ...": recent tokens kept at higher precision).
 *
 * Per-channel key groups (k_per_channel = 1; [P1] "Granularitas ...": the
 * grouping axis may run along token positions): a key group is k_group
 * consecutive positions of one channel, aligned to k_group inside a page.
 * Key codes are then stored like value codes (channel runs of P*kb/8 bytes,
 * chunk-major) and key metadata as
 *   k_meta  [pages][Hkv][P/kg][d] {u16 scale, u16 zero}.
 * A group is quantized only when complete and out of the W newest
 * positions, so positions [0, Q) live in pages with
 * Q = kg * floor(max(0, L-W) / kg), the rest (at most W + kg - 1
 * positions) in a ring of W + kg - 1 slots (slot = position mod (W + kg - 1)):
 * the bf16 window is the residual buffer.
 * ---------------------------------------------------------------------- */
typedef struct {
    int head_dim, num_q_heads, num_kv_heads;
    int k_bits, v_bits, k_group, v_group, page_size, window;
    int rotate_keys;
    const int8_t* rot_signs;       /* host [head_dim] */
    int k_per_channel;             /* 1: key groups run along positions */
} kvqo_layout;

typedef struct {
    uint8_t *k_codes, *v_codes, *k_meta, *v_meta;
    uint16_t *k_win, *v_win;       /* bf16 bit patterns */
    const int32_t* page_table;
    int batch, max_pages_per_seq;
} kvqo_cache;

static int valid_bits(int b) { return b == 1 || b == 2 || b == 4 || b == 8; }

static int check_layout(const kvqo_layout* l)
{
    if (!l) return KVQO_ERR_ARG;
    if (l->head_dim <= 0 || l->head_dim > 256) return KVQO_ERR_UNSUPPORTED;
    if (!valid_bits(l->k_bits) || !valid_bits(l->v_bits)) return KVQO_ERR_UNSUPPORTED;
    if (l->k_group <= 0 || l->v_group <= 0) return KVQO_ERR_UNSUPPORTED;
    if (l->head_dim % l->v_group) return KVQO_ERR_UNSUPPORTED;
    if (l->k_per_channel) {
        if (l->page_size <= 0 || l->page_size % l->k_group || l->k_group > 64) return KVQO_ERR_UNSUPPORTED;
        if ((l->page_size * l->k_bits) % 32 || l->rotate_keys) return KVQO_ERR_UNSUPPORTED;
    } else {
        if (l->head_dim % l->k_group) return KVQO_ERR_UNSUPPORTED;
        if ((l->head_dim * l->k_bits) % 32) return KVQO_ERR_UNSUPPORTED;
    }
    if (l->page_size <= 0 || (l->page_size * l->v_bits) % 32) return KVQO_ERR_UNSUPPORTED;
    if (l->num_kv_heads <= 0 || l->num_q_heads % l->num_kv_heads) return KVQO_ERR_UNSUPPORTED;
    if (l->window < 0) return KVQO_ERR_ARG;
    if (l->rotate_keys && (l->head_dim & (l->head_dim - 1))) return KVQO_ERR_UNSUPPORTED;
    return KVQO_OK;
}

/* bytes of one page of each array ([P1] "Pertumbuhan cache ...": payload
 * plus quantization metadata) */
int kvqo_page_bytes(const kvqo_layout* l, size_t* kc, size_t* km, size_t* vc, size_t* vm)
{
    int rc = check_layout(l);
    if (rc) return rc;
    size_t per = (size_t)l->num_kv_heads * l->page_size;
    *kc = per * (size_t)(l->head_dim * l->k_bits / 8);
    *km = l->k_per_channel
              ? (size_t)l->num_kv_heads * (size_t)(l->page_size / l->k_group) * (size_t)l->head_dim * 4
              : per * (size_t)(l->head_dim / l->k_group) * 4;
    *vc = per * (size_t)(l->head_dim * l->v_bits / 8);
    *vm = per * (size_t)(l->head_dim / l->v_group) * 4;
    return KVQO_OK;
}

static size_t krow_bytes(const kvqo_layout* l) { return (size_t)l->head_dim * l->k_bits / 8; }
static size_t vrow_bytes(const kvqo_layout* l) { return (size_t)l->page_size * l->v_bits / 8; }
static size_t kchan_bytes(const kvqo_layout* l) { return (size_t)l->page_size * l->k_bits / 8; }

/* ring slots of the bf16 window, and the number of positions of a length-L
 * sequence that live in pages */
static int ring_slots(const kvqo_layout* l) { return l->window + (l->k_per_channel ? l->k_group - 1 : 0); }
static int paged_len(const kvqo_layout* l, int L)
{
    int q = L - l->window > 0 ? L - l->window : 0;
    if (l->k_per_channel) q -= q % l->k_group;
    return q;
}

/* Code rows longer than 16 bytes are stored in 16-byte chunks, chunk-major
 * inside the (page, kv-head) block: chunk i of token slot t of a key block
 * sits at i*(P*16) + t*16 (and chunk i of value channel j at i*(d*16) +
 * j*16).  Rows of at most 16 bytes are a single chunk. */
static size_t chunk_of(size_t row_bytes) { return row_bytes < 16 ? row_bytes : 16; }

static uint8_t* k_block(const kvqo_layout* l, const kvqo_cache* c, int page, int h)
{
    return c->k_codes + ((size_t)page * l->num_kv_heads + h) * (size_t)l->page_size * krow_bytes(l);
}
static uint8_t* v_block(const kvqo_layout* l, const kvqo_cache* c, int page, int h)
{
    return c->v_codes + ((size_t)page * l->num_kv_heads + h) * (size_t)l->head_dim * vrow_bytes(l);
}
/* gather (put = 0) or scatter (put = 1) the packed key row of one token */
static void k_row_io(const kvqo_layout* l, const kvqo_cache* c, int page, int h, int slot,
                     uint8_t* row, int put)
{
    size_t rb = krow_bytes(l), ch = chunk_of(rb);
    uint8_t* base = k_block(l, c, page, h);
    for (size_t i = 0; i < rb / ch; ++i) {
        uint8_t* at = base + i * (size_t)l->page_size * ch + (size_t)slot * ch;
        if (put) memcpy(at, row + i * ch, ch);
        else memcpy(row + i * ch, at, ch);
    }
}
/* gather or scatter the packed token run of one value channel */
static void v_chan_io(const kvqo_layout* l, const kvqo_cache* c, int page, int h, int j,
                      uint8_t* run, int put)
{
    size_t rb = vrow_bytes(l), ch = chunk_of(rb);
    uint8_t* base = v_block(l, c, page, h);
    for (size_t i = 0; i < rb / ch; ++i) {
        uint8_t* at = base + i * (size_t)l->head_dim * ch + (size_t)j * ch;
        if (put) memcpy(at, run + i * ch, ch);
        else memcpy(run + i * ch, at, ch);
    }
}
/* per-channel keys: gather or scatter the packed token run of key channel j */
static void k_chan_io(const kvqo_layout* l, const kvqo_cache* c, int page, int h, int j,
                      uint8_t* run, int put)
{
    size_t rb = kchan_bytes(l), ch = chunk_of(rb);
    uint8_t* base = k_block(l, c, page, h);
    for (size_t i = 0; i < rb / ch; ++i) {
        uint8_t* at = base + i * (size_t)l->head_dim * ch + (size_t)j * ch;
        if (put) memcpy(at, run + i * ch, ch);
        else memcpy(run + i * ch, at, ch);
    }
}
/* per-channel keys: metadata of group grp (slots grp*kg ..) of channel j */
static uint8_t* k_meta_chan(const kvqo_layout* l, const kvqo_cache* c, int page, int h, int grp, int j)
{
    return c->k_meta + ((((size_t)page * l->num_kv_heads + h) * (size_t)(l->page_size / l->k_group) + grp) *
                            (size_t)l->head_dim + j) * 4;
}
static uint8_t* k_meta_row(const kvqo_layout* l, const kvqo_cache* c, int page, int h, int slot)
{
    return c->k_meta + (((size_t)page * l->num_kv_heads + h) * l->page_size + slot) *
                           (size_t)(l->head_dim / l->k_group) * 4;
}
static uint8_t* v_meta_row(const kvqo_layout* l, const kvqo_cache* c, int page, int h, int slot)
{
    return c->v_meta + (((size_t)page * l->num_kv_heads + h) * l->page_size + slot) *
                           (size_t)(l->head_dim / l->v_group) * 4;
}
static uint16_t* win_row(const kvqo_layout* l, uint16_t* win, int b, int h, int pos)
{
    const int R = ring_slots(l);
    return win + (((size_t)b * l->num_kv_heads + h) * R + (size_t)(pos % R)) * l->head_dim;
}

static void put_meta(uint8_t* m, uint16_t scale, uint16_t zero)
{
    m[0] = (uint8_t)scale; m[1] = (uint8_t)(scale >> 8);
    m[2] = (uint8_t)zero;  m[3] = (uint8_t)(zero >> 8);
}
static void get_meta(const uint8_t* m, uint16_t* scale, uint16_t* zero)
{
    *scale = (uint16_t)(m[0] | (m[1] << 8));
    *zero = (uint16_t)(m[2] | (m[3] << 8));
}

/* quantize the value row of one token of one kv-head into its page slot:
 * groups of v_group channels, codes stored per channel */
static void quantize_token_values(const kvqo_layout* l, const kvqo_cache* c, int b, int h,
                                  int pos, const float* v)
{
    int d = l->head_dim;
    int page = c->page_table[(size_t)b * c->max_pages_per_seq + pos / l->page_size];
    int slot = pos % l->page_size;
    uint8_t codes[256];
    uint8_t* vm = v_meta_row(l, c, page, h, slot);
    for (int g = 0; g < d / l->v_group; ++g) {
        uint16_t s, z;
        kvqo_quantize_group(v + g * l->v_group, l->v_group, l->v_bits, &s, &z,
                            codes + g * l->v_group);
        put_meta(vm + 4 * g, s, z);
    }
    for (int j = 0; j < d; ++j) {
        uint8_t run[64];
        v_chan_io(l, c, page, h, j, run, 0);
        set_packed(run, slot, l->v_bits, codes[j]);
        v_chan_io(l, c, page, h, j, run, 1);
    }
}

/* quantize one token of one kv-head (fp32 k, v) into its page slot; keys in
 * groups of k_group channels (rotated first when the layout rotates keys) */
static void quantize_token(const kvqo_layout* l, const kvqo_cache* c, int b, int h,
                           int pos, const float* k, const float* v)
{
    int d = l->head_dim;
    int page = c->page_table[(size_t)b * c->max_pages_per_seq + pos / l->page_size];
    int slot = pos % l->page_size;
    float kr[256];
    uint8_t codes[256];
    if (l->rotate_keys) kvqo_rotate(k, l->rot_signs, d, kr);
    else memcpy(kr, k, sizeof(float) * d);
    uint8_t* km = k_meta_row(l, c, page, h, slot);
    for (int g = 0; g < d / l->k_group; ++g) {
        uint16_t s, z;
        kvqo_quantize_group(kr + g * l->k_group, l->k_group, l->k_bits, &s, &z,
                            codes + g * l->k_group);
        put_meta(km + 4 * g, s, z);
    }
    uint8_t row[256];
    kvqo_pack(codes, d, l->k_bits, row);
    k_row_io(l, c, page, h, slot, row, 1);
    quantize_token_values(l, c, b, h, pos, v);
}

/* per-channel keys: quantize the keys of positions [g0, g0 + k_group) of
 * (b, kv-head h), K [k_group][d] fp32; one group per channel */
static void quantize_key_group(const kvqo_layout* l, const kvqo_cache* c, int b, int h,
                               int g0, const float* K)
{
    const int d = l->head_dim, G = l->k_group;
    int page = c->page_table[(size_t)b * c->max_pages_per_seq + g0 / l->page_size];
    int slot0 = g0 % l->page_size;
    for (int j = 0; j < d; ++j) {
        float x[64];
        uint8_t codes[64], run[64];
        uint16_t s, z;
        for (int t = 0; t < G; ++t) x[t] = K[(size_t)t * d + j];
        kvqo_quantize_group(x, G, l->k_bits, &s, &z, codes);
        put_meta(k_meta_chan(l, c, page, h, slot0 / G, j), s, z);
        k_chan_io(l, c, page, h, j, run, 0);
        for (int t = 0; t < G; ++t) set_packed(run, slot0 + t, l->k_bits, codes[t]);
        k_chan_io(l, c, page, h, j, run, 1);
    }
}

static float load_in(const void* p, int in_dtype, size_t idx)
{
    if (in_dtype == 1) return kvqo_bf16_to_f32(((const uint16_t*)p)[idx]);
    return ((const float*)p)[idx];
}

/* Append new tokens (ragged rows [total_new][Hkv][d], row offsets cu_new)
 * after lens[b] existing positions.  Positions that leave the bf16 window
 * ([P1] "Pertumbuhan cache ...") are quantized into pages; the newest
 * min(W, L+n) positions are kept in the ring.  in_dtype: 0 = fp32,
 * 1 = bf16.  fp32 rows entering the bf16 ring are rounded to nearest even.
 */
int kvqo_quantize_append(const kvqo_layout* l, const kvqo_cache* c,
                         const void* k_new, const void* v_new, int in_dtype,
                         const int32_t* cu_new, const int32_t* lens)
{
    int rc = check_layout(l);
    if (rc) return rc;
    if (!c || !k_new || !v_new || !cu_new || !lens) return KVQO_ERR_ARG;
    const int d = l->head_dim, H = l->num_kv_heads;
    int B = c->batch;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        int L = lens[b];
        int n = cu_new[b + 1] - cu_new[b];
        int q0 = paged_len(l, L), q1 = paged_len(l, L + n);
        /* fp32 row of position pos (< L + n) of (b, h): the ring when older than L */
        #define KVQO_ROW(pos, h, kdst, vdst)                                              \
            do {                                                                          \
                if ((pos) < L) {                                                          \
                    uint16_t* kw_ = win_row(l, c->k_win, b, (h), (pos));                  \
                    uint16_t* vw_ = win_row(l, c->v_win, b, (h), (pos));                  \
                    for (int j_ = 0; j_ < d; ++j_) {                                      \
                        (kdst)[j_] = kvqo_bf16_to_f32(kw_[j_]);                           \
                        (vdst)[j_] = kvqo_bf16_to_f32(vw_[j_]);                           \
                    }                                                                     \
                } else {                                                                  \
                    size_t row_ = ((size_t)(cu_new[b] + (pos) - L) * H + (h)) * d;       \
                    for (int j_ = 0; j_ < d; ++j_) {                                      \
                        (kdst)[j_] = load_in(k_new, in_dtype, row_ + j_);                 \
                        (vdst)[j_] = load_in(v_new, in_dtype, row_ + j_);                 \
                    }                                                                     \
                }                                                                         \
            } while (0)
        if (!l->k_per_channel) {
            /* every position that leaves the window (or never enters it) */
            float k[256], v[256];
            for (int pos = q0; pos < q1; ++pos)
                for (int h = 0; h < H; ++h) {
                    KVQO_ROW(pos, h, k, v);
                    quantize_token(l, c, b, h, pos, k, v);
                }
        } else {
            /* every key group that became complete and left the window */
            const int G = l->k_group;
            float* K = (float*)malloc(sizeof(float) * (size_t)G * d);
            float v[256];
            for (int g0 = q0; g0 < q1; g0 += G)
                for (int h = 0; h < H; ++h) {
                    for (int t = 0; t < G; ++t) {
                        KVQO_ROW(g0 + t, h, K + (size_t)t * d, v);
                        quantize_token_values(l, c, b, h, g0 + t, v);
                    }
                    quantize_key_group(l, c, b, h, g0, K);
                }
            free(K);
        }
        #undef KVQO_ROW
        /* the new positions that stay in the window go to the ring (after
         * the reads above: a slot may be reused) */
        if (ring_slots(l) > 0) {
            int w0 = q1 > L ? q1 : L;
            for (int pos = w0; pos < L + n; ++pos) {
                for (int h = 0; h < H; ++h) {
                    size_t row = ((size_t)(cu_new[b] + pos - L) * H + h) * d;
                    uint16_t* kw = win_row(l, c->k_win, b, h, pos);
                    uint16_t* vw = win_row(l, c->v_win, b, h, pos);
                    for (int j = 0; j < d; ++j) {
                        if (in_dtype == 1) {
                            kw[j] = ((const uint16_t*)k_new)[row + j];
                            vw[j] = ((const uint16_t*)v_new)[row + j];
                        } else {
                            kw[j] = kvqo_f32_to_bf16(((const float*)k_new)[row + j], KVQO_RN);
                            vw[j] = kvqo_f32_to_bf16(((const float*)v_new)[row + j], KVQO_RN);
                        }
                    }
                }
            }
        }
    }
    return KVQO_OK;
}

/* Reconstruct position pos of (b, kv-head h): keys (rotated domain when the
 * layout rotates keys and pos is quantized) and values, fp32. Returns 1 if
 * the position is quantized, 0 if it comes from the bf16 window. */
static int reconstruct(const kvqo_layout* l, const kvqo_cache* c, int b, int h,
                       int L, int pos, float* k, float* v)
{
    int d = l->head_dim;
    if (pos >= paged_len(l, L)) {
        const uint16_t* kw = win_row(l, c->k_win, b, h, pos);
        const uint16_t* vw = win_row(l, c->v_win, b, h, pos);
        for (int j = 0; j < d; ++j) {
            k[j] = kvqo_bf16_to_f32(kw[j]);
            v[j] = kvqo_bf16_to_f32(vw[j]);
        }
        return 0;
    }
    int page = c->page_table[(size_t)b * c->max_pages_per_seq + pos / l->page_size];
    int slot = pos % l->page_size;
    uint8_t kc[256], vrun[64], krun[64];
    if (!l->k_per_channel) k_row_io(l, c, page, h, slot, kc, 0);
    const uint8_t* km = k_meta_row(l, c, page, h, slot);
    const uint8_t* vm = v_meta_row(l, c, page, h, slot);
    for (int j = 0; j < d; ++j) {
        uint16_t s, z;
        if (l->k_per_channel) {
            k_chan_io(l, c, page, h, j, krun, 0);
            get_meta(k_meta_chan(l, c, page, h, slot / l->k_group, j), &s, &z);
            k[j] = kvqo_dequant_code(kvqo_unpack_one(krun, slot, l->k_bits), s, z);
        } else {
            get_meta(km + 4 * (j / l->k_group), &s, &z);
            k[j] = kvqo_dequant_code(kvqo_unpack_one(kc, j, l->k_bits), s, z);
        }
        get_meta(vm + 4 * (j / l->v_group), &s, &z);
        v_chan_io(l, c, page, h, j, vrun, 0);
        v[j] = kvqo_dequant_code(kvqo_unpack_one(vrun, slot, l->v_bits), s, z);
    }
    return 1;
}

/* Reconstructed cache, fp32 [B][Hkv][max_len][d]; positions >= lens[b] are
 * left untouched ([P1] "Pertumbuhan cache ...": dequantization to temporary
 * storage is one of the serving paths). */
int kvqo_dequantize(const kvqo_layout* l, const kvqo_cache* c, const int32_t* lens,
                    int max_len, float* k_out, float* v_out)
{
    int rc = check_layout(l);
    if (rc) return rc;
    const int d = l->head_dim, H = l->num_kv_heads, B = c->batch;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            int L = lens[b] < max_len ? lens[b] : max_len;
            for (int pos = 0; pos < L; ++pos) {
                size_t o = (((size_t)b * H + h) * max_len + pos) * d;
                reconstruct(l, c, b, h, lens[b], pos, k_out + o, v_out + o);
            }
        }
    return KVQO_OK;
}

/* ------------------------------------------------------------------------
 * Attention in fp64 ([P1] "Error pada key masuk sebelum softmax"):
 * s = q K^T * sm_scale, a = softmax(s), o = a V, plus lse = log sum exp(s).
 * q [d], K and V [L][d] dense.  L = 0 gives o = 0 and lse = -inf.
 * ---------------------------------------------------------------------- */
void kvqo_attention_dense(const double* q, const double* K, const double* V,
                          int L, int d, double sm_scale, double* o, double* lse)
{
    for (int j = 0; j < d; ++j) o[j] = 0.0;
    if (L <= 0) {
        *lse = -INFINITY;
        return;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)L);
    double mx = -INFINITY;
    for (int t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += q[j] * K[(size_t)t * d + j];
        s[t] = acc * sm_scale;
        if (s[t] > mx) mx = s[t];
    }
    double sum = 0.0;
    for (int t = 0; t < L; ++t) {
        s[t] = exp(s[t] - mx);
        sum += s[t];
    }
    for (int t = 0; t < L; ++t) {
        double a = s[t] / sum;
        for (int j = 0; j < d; ++j) o[j] += a * V[(size_t)t * d + j];
    }
    *lse = mx + log(sum);
    free(s);
}

/* Softmax attention of one query over positions [0, n) of the reconstructed
 * rows K, V [n][d] of one (sequence, kv-head), fp64 ([P1] "Error pada key
 * masuk sebelum softmax": s = q K^T * sm_scale, a = softmax(s), o = a V,
 * lse = log sum exp(s)).  Quantized keys of a rotating layout are in the
 * rotated domain, so rows with quant[t] set are scored with the rotated
 * query qr; the other rows (bf16 window) with the plain query qd. */
static void attend_prefix(const kvqo_layout* l, const double* qd, const double* qr,
                          const double* K, const double* V, const int* quant, int n,
                          double sm_scale, double* o, double* lo)
{
    const int d = l->head_dim;
    if (!l->rotate_keys) {
        kvqo_attention_dense(qd, K, V, n, d, sm_scale, o, lo);
        return;
    }
    for (int j = 0; j < d; ++j) o[j] = 0.0;
    if (n <= 0) { *lo = -INFINITY; return; }
    double* s = (double*)malloc(sizeof(double) * (size_t)n);
    double mx = -INFINITY, sum = 0.0;
    for (int t = 0; t < n; ++t) {
        const double* qq = quant[t] ? qr : qd;
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += qq[j] * K[(size_t)t * d + j];
        s[t] = acc * sm_scale;
        if (s[t] > mx) mx = s[t];
    }
    for (int t = 0; t < n; ++t) { s[t] = exp(s[t] - mx); sum += s[t]; }
    for (int t = 0; t < n; ++t) {
        double a = s[t] / sum;
        for (int j = 0; j < d; ++j) o[j] += a * V[(size_t)t * d + j];
    }
    *lo = mx + log(sum);
    free(s);
}

/* Reconstruct positions [0, L) of (b, kv-head h) into K, V [L][d] (fp64) and
 * quant[L] (1 = from a page, 0 = from the bf16 window). */
static void reconstruct_all(const kvqo_layout* l, const kvqo_cache* c, int b, int h, int L,
                            double* K, double* V, int* quant)
{
    const int d = l->head_dim;
    float kf[256], vf[256];
    for (int pos = 0; pos < L; ++pos) {
        quant[pos] = reconstruct(l, c, b, h, L, pos, kf, vf);
        for (int j = 0; j < d; ++j) {
            K[(size_t)pos * d + j] = kf[j];
            V[(size_t)pos * d + j] = vf[j];
        }
    }
}

/* query row (fp64) of q-head hq of query row r of q [rows][Hq][d], and its
 * rotation when the layout rotates keys */
static void load_query(const kvqo_layout* l, const void* q, int q_dtype, size_t r, int hq,
                       double* qd, double* qr)
{
    const int d = l->head_dim, Hq = l->num_q_heads;
    for (int j = 0; j < d; ++j) qd[j] = load_in(q, q_dtype, (r * Hq + hq) * d + j);
    if (l->rotate_keys) kvqo_rotate_f64(qd, l->rot_signs, d, qr);
}

/* Decode attention of one query token per sequence over the cache, fp64.
 * q [B][Hq][d] (q_dtype 0 = fp32, 1 = bf16); query head hq reads kv-head
 * hq / (Hq/Hkv).  out [B][Hq][d], lse [B][Hq] (natural log). */
int kvqo_decode_attention(const kvqo_layout* l, const kvqo_cache* c, const void* q,
                          int q_dtype, const int32_t* lens, double sm_scale,
                          double* out, double* lse)
{
    int rc = check_layout(l);
    if (rc) return rc;
    const int d = l->head_dim, H = l->num_kv_heads, Hq = l->num_q_heads, B = c->batch;
    const int g = Hq / H;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            int L = lens[b];
            double* K = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * d);
            double* V = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * d);
            int* quant = (int*)malloc(sizeof(int) * (size_t)(L > 0 ? L : 1));
            reconstruct_all(l, c, b, h, L, K, V, quant);
            for (int r = 0; r < g; ++r) {
                int hq = h * g + r;
                double qd[256], qr[256];
                load_query(l, q, q_dtype, (size_t)b, hq, qd, qr);
                attend_prefix(l, qd, qr, K, V, quant, L, sm_scale,
                              out + ((size_t)b * Hq + hq) * d, lse + (size_t)b * Hq + hq);
            }
            free(K); free(V); free(quant);
        }
    return KVQO_OK;
}

/* Attention of a chunk of new query tokens over the cache (chunked prefill),
 * causal, fp64.  The chunk's own keys and values were appended first, so
 * sequence b holds lens[b] positions and its n_b = cu_q[b+1] - cu_q[b]
 * queries are the newest n_b positions: query i sits at position
 * p = lens[b] - n_b + i and attends to positions [0, p] as the cache holds
 * them now (pages or bf16 window; [P1] "Pertumbuhan cache ...": the stored
 * approximation is what later attention reads).  The pages describe one new
 * query; extending it to a chunk with a causal mask is the plain reading.
 * q [total_q][Hq][d] rows cu_q[b] + i; out [total_q][Hq][d],
 * lse [total_q][Hq].  n_b < 0 or n_b > lens[b] is an argument error. */
int kvqo_prefill_attention(const kvqo_layout* l, const kvqo_cache* c, const void* q,
                           int q_dtype, const int32_t* cu_q, const int32_t* lens,
                           double sm_scale, double* out, double* lse)
{
    int rc = check_layout(l);
    if (rc) return rc;
    const int d = l->head_dim, H = l->num_kv_heads, Hq = l->num_q_heads, B = c->batch;
    const int g = Hq / H;
    for (int b = 0; b < B; ++b) {
        int n = cu_q[b + 1] - cu_q[b];
        if (n < 0 || n > lens[b]) return KVQO_ERR_ARG;
    }
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            int L = lens[b], n = cu_q[b + 1] - cu_q[b];
            if (n == 0) continue;
            double* K = (double*)malloc(sizeof(double) * (size_t)L * d);
            double* V = (double*)malloc(sizeof(double) * (size_t)L * d);
            int* quant = (int*)malloc(sizeof(int) * (size_t)L);
            reconstruct_all(l, c, b, h, L, K, V, quant);
            for (int i = 0; i < n; ++i) {
                size_t row = (size_t)cu_q[b] + i;
                int visible = L - n + i + 1;
                for (int r = 0; r < g; ++r) {
                    int hq = h * g + r;
                    double qd[256], qr[256];
                    load_query(l, q, q_dtype, row, hq, qd, qr);
                    attend_prefix(l, qd, qr, K, V, quant, visible, sm_scale,
                                  out + (row * Hq + hq) * d, lse + row * Hq + hq);
                }
            }
            free(K); free(V); free(quant);
        }
    return KVQO_OK;
}

int kvqo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void kvqo_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------
 * Array forms of the scalar helpers above (plain loops), so the tests can
 * sweep millions of inputs without one foreign call per element.
 * ---------------------------------------------------------------------- */
void kvqo_f32_to_f16_n(const float* x, long n, int mode, uint16_t* out)
{
    for (long i = 0; i < n; ++i) out[i] = kvqo_f32_to_f16(x[i], mode);
}

void kvqo_f32_to_bf16_n(const float* x, long n, int mode, uint16_t* out)
{
    for (long i = 0; i < n; ++i) out[i] = kvqo_f32_to_bf16(x[i], mode);
}

void kvqo_op_n(const float* a, const float* b, long n, int op, int up, float* out)
{
    for (long i = 0; i < n; ++i) {
        if (op == 0) out[i] = up ? kvqo_sub_ru(a[i], b[i]) : kvqo_sub_rn(a[i], b[i]);
        else out[i] = up ? kvqo_div_ru(a[i], b[i]) : kvqo_div_rn(a[i], b[i]);
    }
}

/* rows of row_len values, groups of `group` contiguous values */
void kvqo_quantize_rows(const float* x, long rows, int row_len, int group, int bits,
                        uint16_t* scale, uint16_t* zero, uint8_t* codes)
{
    int ng = row_len / group;
    for (long r = 0; r < rows; ++r)
        for (int g = 0; g < ng; ++g)
            kvqo_quantize_group(x + r * row_len + g * group, group, bits,
                                scale + r * ng + g, zero + r * ng + g,
                                codes + r * row_len + g * group);
}

void kvqo_dequantize_rows(const uint8_t* codes, const uint16_t* scale, const uint16_t* zero,
                          long rows, int row_len, int group, float* out)
{
    int ng = row_len / group;
    for (long r = 0; r < rows; ++r)
        for (int j = 0; j < row_len; ++j)
            out[r * row_len + j] = kvqo_dequant_code(codes[r * row_len + j],
                                                     scale[r * ng + j / group],
                                                     zero[r * ng + j / group]);
}

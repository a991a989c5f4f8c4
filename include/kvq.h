/*
 * kvq.h -- C ABI of the B200 (sm_100a) mixed-precision quantized KV cache.
 *
 * What it computes (sources are web pages, cited by title and section):
 *  - "Kuantisasi KV cache mengganggu attention melalui key dan value
 *    tersimpan" (nalar.dev), section "Error pada key masuk sebelum softmax":
 *    decode attention s = q K^T * sm_scale, a = softmax(s), o = a V over the
 *    stored (reconstructed) keys and values; section "Granularitas
 *    kuantisasi menentukan nilai yang berbagi scale": a group of values
 *    shares one scale and one zero point; section "Pertumbuhan cache
 *    mengubah trade pada serving": the newest tokens stay at higher
 *    precision while older ones are quantized, and dequantization can be
 *    fused into the attention kernel or done into temporary storage.
 *  - "Quantize What Counts: More for Keys, Less for Values" (summary of
 *    arXiv 2502.15075), Methodologie / Belangrijkste Bijdragen / Resultaten:
 *    more bits for keys than values (e.g. K4V2), key groups of 32 channels,
 *    value groups of 64-128, optional rotation of keys only.
 *
 * Quantizer (per token, per group of contiguous channels; the pages print
 * no formula, this is the min/max reading):
 *    zero  = fp16 of min(x) rounded toward -inf
 *    scale = fp16 of ((max(x) - zero) / (2^b - 1)), every step rounded up
 *    code  = clamp(rint((x - zero) / scale), 0, 2^b - 1)   (ties to even)
 *    x^    = code * scale + zero                           (one fp32 fma)
 * so |x - x^| <= scale/2 (+ fp32 rounding) for every element.  Inputs must
 * keep group minima >= -65504 and (max - zero)/(2^b - 1) <= 65504; NaN and
 * Inf are not supported.
 *
 * Conventions for every entry point:
 *  - Device buffers are owned by the caller; the library never allocates,
 *    frees or synchronizes, and keeps no pointer after a call returns.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  Calls on one stream run in order.
 *  - Return value: KVQ_OK, or a negative KVQ_ERR_* code.  Arguments are
 *    checked on the host before anything is launched; on an error nothing
 *    is enqueued.  KVQ_ERR_CUDA reports a failed launch.
 *  - Lengths live on the device (int32).  The host passes an upper bound
 *    (max_len / max_new) used to size the launch; device lengths above it
 *    are clamped to it, and page-table entries outside [0, num_pages) are
 *    treated as absent pages (their tokens are skipped, never read).
 *
 * Storage layout (P = page_size tokens, d = head_dim, per layer):
 *    k_codes [num_pages][Hkv][P][d*k_bits/8]  token rows; channel j in bits
 *            k_bits*(j mod (32/k_bits)) of little-endian 32-bit word
 *            floor(j*k_bits/32)
 *    k_meta  [num_pages][Hkv][P][d/k_group] x {uint16 scale, uint16 zero}
 *            (IEEE binary16 bit patterns)
 *    v_codes [num_pages][Hkv][d][P*v_bits/8]  channel rows; token slot t in
 *            bits v_bits*(t mod (32/v_bits)) of word floor(t*v_bits/32)
 *    v_meta  [num_pages][Hkv][P][d/v_group] x {uint16 scale, uint16 zero}
 *    k_win, v_win [batch][Hkv][window][d] bf16 ring, slot = position % window
 *    page_table [batch][max_pages_per_seq] int32 physical page ids
 *  Code rows longer than 16 bytes (key rows of d*k_bits/8 bytes, value
 *  channel runs of P*v_bits/8 bytes) are stored as 16-byte chunks,
 *  chunk-major inside each (page, kv-head) block: chunk i of token slot t
 *  at byte i*(P*16) + t*16 of the key block, chunk i of channel j at byte
 *  i*(d*16) + j*16 of the value block.  A row of at most 16 bytes is one
 *  chunk, so the plain row-major form above is then exact.
 *  Position p of sequence b lives in page page_table[b][p / P], slot p % P,
 *  when p < len - window, and in ring slot p % window otherwise.  All
 *  buffers must be 16-byte aligned.
 *
 * Per-channel key groups (k_per_channel = 1; "Granularitas kuantisasi
 * ...": the grouping axis may run along token positions): a key group is
 * k_group consecutive positions of ONE channel, aligned to k_group inside
 * a page, quantized with the same min/max rule.  Then
 *    k_codes [num_pages][Hkv][d][P*k_bits/8]  channel runs, stored like
 *            v_codes (token slot t in bits k_bits*(t mod (32/k_bits)) of
 *            word floor(t*k_bits/32); chunk-major above 16 bytes)
 *    k_meta  [num_pages][Hkv][P/k_group][d] x {uint16 scale, uint16 zero}
 *    k_win, v_win [batch][Hkv][window + k_group - 1][d] bf16 ring, slot =
 *            position % (window + k_group - 1)
 *  A key group is quantized once it is complete and out of the window
 *  newest positions, so positions below Q = k_group*floor(max(0, len -
 *  window)/k_group) live in pages and the rest (window to window +
 *  k_group - 1 positions) in the ring.  Values keep per-token groups.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kvq_stream_t; /* same type as cudaStream_t */

enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = -1,  /* null pointer, negative size, bad alignment */
    KVQ_ERR_UNSUPPORTED = -2,  /* bits, head_dim, groups or GQA outside the supported set */
    KVQ_ERR_WORKSPACE = -3,    /* workspace missing or smaller than kvq_decode_workspace_bytes */
    KVQ_ERR_CUDA = -4          /* a CUDA call or launch failed */
};

enum { KVQ_F32 = 0, KVQ_BF16 = 1 }; /* element types of inputs */

/* Problem statement of one layer's cache.
 * head_dim        d, 64 or 128
 * num_q_heads     Hq; num_kv_heads Hkv; Hq % Hkv == 0, 1 <= Hq/Hkv <= 8
 *                 (query head h reads kv-head h / (Hq/Hkv))
 * k_bits, v_bits  1, 2, 4 or 8 ("more for keys": k_bits >= v_bits is the
 *                 intended use, not a requirement)
 * k_group,v_group channels per group: 16, 32, 64 or 128, dividing d
 *                 (with k_per_channel, k_group counts positions: 16, 32
 *                 or 64)
 * page_size       tokens per page: 64
 * window          W >= 0 newest positions kept in bf16 (0 = none)
 * rotate_keys     1 = keys are multiplied by (diag(rot_signs) H / sqrt(d))
 *                 before quantization (H Sylvester Walsh-Hadamard) and the
 *                 query is rotated the same way when scoring quantized
 *                 positions; window keys stay unrotated.
 * rot_signs       device int8 [d] of +1/-1, required when rotate_keys
 * k_per_channel   1 = key groups run along positions of one channel (see
 *                 the storage layout above); not combined with
 *                 rotate_keys.  Decode and prefill attention then run on
 *                 CUDA cores and need no workspace.
 */
typedef struct kvq_layout {
    int head_dim;
    int num_q_heads;
    int num_kv_heads;
    int k_bits;
    int v_bits;
    int k_group;
    int v_group;
    int page_size;
    int window;
    int rotate_keys;
    const int8_t* rot_signs;
    int k_per_channel;
} kvq_layout;

/* Device buffers of one layer's cache (layout in the file header). */
typedef struct kvq_cache {
    void* k_codes;
    void* v_codes;
    void* k_meta;
    void* v_meta;
    void* k_win;                 /* bf16; may be NULL when window == 0 */
    void* v_win;
    const int32_t* page_table;   /* device [batch][max_pages_per_seq] */
    int batch;
    int max_pages_per_seq;
    int num_pages;               /* physical pages in k_codes/... */
} kvq_cache;

/* Message for a status code (static string, never NULL). */
const char* kvq_status_string(int status);

/* Library version: major*10000 + minor*100 + patch. */
int kvq_version(void);

/* Bytes of ONE physical page of each array (all kv-heads of the page):
 * codes plus fp16 metadata ("Pertumbuhan cache ...": memory = payload +
 * metadata).  Any output pointer may be NULL. */
int kvq_page_bytes(const kvq_layout* layout, size_t* k_codes, size_t* k_meta,
                   size_t* v_codes, size_t* v_meta);

/* Bytes of one window ring (k_win or v_win) for `batch` sequences. */
int kvq_window_bytes(const kvq_layout* layout, int batch, size_t* bytes);

/* Workspace that kvq_decode_attention needs for this batch and bound on
 * lengths on the current device (split partials); 0 on invalid input, and
 * for k_per_channel layouts the bytes that let the decode split each (sequence,
 * kv-head) between CTAs when the pairs leave SMs idle, else 0; for these
 * layouts the workspace is optional (NULL, or smaller: one CTA per pair). */
size_t kvq_decode_workspace_bytes(const kvq_layout* layout, int batch, int max_len);

/* Select the decode kernel family for subsequent kvq_decode_attention and
 * kvq_decode_workspace_bytes calls (process-wide):
 *   0  automatic (default): the persistent tensor-core kernel where the
 *      layout supports it (head_dim 128, key groups of 32, value groups of
 *      128, any key and value bit widths, batch <= 4096), the CUDA-core
 *      kernel otherwise
 *   1  CUDA-core kernel for every layout
 *   2  same as 0 (tensor cores where supported)
 *   3  the two-phase tcgen05 kernel with a separate combine launch where the
 *      layout supports it (same layouts, any batch), CUDA cores otherwise
 * Not thread-safe with concurrent calls; query workspace sizes after
 * changing it.  Returns KVQ_ERR_INVALID_ARG for other values. */
int kvq_set_decode_path(int path);

/* Decode kernel family the current setting picks for this layout (at batch
 * 1, short sequences): 2 = persistent tensor-core kernel, 3 = two-phase
 * tcgen05 kernel, 1 = CUDA cores, 4 = the per-channel decode kernel (the
 * k_per_channel layouts it takes: head_dim 128, unrotated; other
 * k_per_channel layouts report 1), or a negative KVQ_ERR_* code.  The
 * setting of kvq_set_decode_path does not apply to k_per_channel layouts. */
int kvq_get_decode_path(const kvq_layout* layout);

/* Decode diagnostics of the current device, counted by the decode kernels
 * since the library was loaded (or last cleared):
 *   wait_timeouts  bounded waits inside a decode kernel that gave up (the
 *                  kernel then writes NaN for the outputs it could not
 *                  finish; 0 in normal operation)
 *   bad_tickets    merge tickets found above their count, i.e. a workspace
 *                  that was not zero-filled before its first use (the
 *                  outputs of those (sequence, kv-head) pairs are not valid)
 * Either pointer may be NULL; clear != 0 resets both counters.  This call
 * reads device memory synchronously (it waits for the device), unlike every
 * other entry point; use it for checking, not inside a timed loop. */
int kvq_decode_status(unsigned int* wait_timeouts, unsigned int* bad_tickets, int clear);

/* Append new tokens and quantize what leaves the bf16 window.
 * ("Granularitas kuantisasi ..." group quantizer; "Pertumbuhan cache ..."
 * recent-token window; "Quantize What Counts" K/V bit split.)
 * k_new, v_new  device [total_new][Hkv][d], in_dtype KVQ_BF16 or KVQ_F32,
 *               rows of sequence b are cu_new[b] .. cu_new[b+1]-1
 * cu_new        device int32 [batch+1], non-decreasing, cu_new[0] == 0
 * lens          device int32 [batch], tokens already in the cache; NOT
 *               updated here -- the caller advances it (lens += n) on the
 *               same stream before the next call
 * max_new       host bound on cu_new[b+1]-cu_new[b] (launch size)
 * Positions [max(0, L-W), max(0, L+n-W)) are quantized into pages (read
 * from the ring when older than L); positions [max(L, L+n-W), L+n) are
 * written to the ring (fp32 input rounded to nearest-even bf16).  Pages
 * must be mapped for every quantized position. */
int kvq_quantize_append(const kvq_layout* layout, const kvq_cache* cache,
                        const void* k_new, const void* v_new, int in_dtype,
                        const int32_t* cu_new, const int32_t* lens, int max_new,
                        kvq_stream_t stream);

/* Decode attention of one query token per sequence over the cache, with
 * dequantization fused into the kernel ("Pertumbuhan cache ..."), GQA and
 * ragged lengths; split-K over the sequence, then a log-sum-exp combine.
 * q         device [batch][Hq][d], q_dtype KVQ_BF16 or KVQ_F32
 * lens      device int32 [batch] (cached tokens); max_len >= max(lens)
 * sm_scale  score scale (1/sqrt(d) for standard attention)
 * out       device fp32 [batch][Hq][d]; lse device fp32 [batch][Hq] (natural
 *           log of sum exp(scores)) or NULL.  A sequence of length 0 gets
 *           out = 0 and lse = -inf.
 * workspace device, >= kvq_decode_workspace_bytes(layout, batch, max_len)
 *           bytes, 256-byte aligned, ZERO-FILLED BEFORE ITS FIRST USE (for
 *           example cudaMemsetAsync after allocating it).  It holds split
 *           partials and one merge ticket per (sequence, kv-head); every
 *           call leaves the tickets at zero again, so the zero fill is needed
 *           once per allocation, not per call.  Calls that overlap on the GPU
 *           need separate workspaces.
 *           Optional for k_per_channel layouts (may be NULL): those run the
 *           per-channel decode kernel, one CTA per (sequence, kv-head) whose
 *           warps merge their parts in shared memory, or, when the workspace
 *           holds kvq_decode_workspace_bytes (zero-filled before its first
 *           use, like the others), several CTAs per pair merged through it
 *           by the last one to finish (head_dim 64 layouts: the
 *           chunked-prefill kernel with one query per sequence).
 * Returns KVQ_ERR_UNSUPPORTED for batch or num_kv_heads above 65535. */
int kvq_decode_attention(const kvq_layout* layout, const kvq_cache* cache,
                         const void* q, int q_dtype, const int32_t* lens, int max_len,
                         float sm_scale, float* out, float* lse,
                         void* workspace, size_t workspace_bytes, kvq_stream_t stream);

/* One decode step: kvq_quantize_append(k_new, v_new, in_dtype, cu_new,
 * lens_old, max_new) followed by kvq_decode_attention(q, q_dtype, lens,
 * max_len, sm_scale, out, lse, workspace) on the same stream, with the same
 * arguments, results and error codes as those two calls (lens_old is the
 * append's `lens`: tokens before the step; lens the decode's: tokens after
 * it, typically lens_old + 1; both stay unmodified).  Not in the pages: it
 * exists so that the decode's start-up overlaps the append.  When the append
 * is one launch (at most 8 new tokens per sequence, and not more than the
 * window) and the persistent tensor-core decode applies, the decode is
 * launched as the append's programmatic dependent: it reads lens, the page
 * table and q while the append runs, and the cache only after the append's
 * results are visible; otherwise the two calls run one after the other.
 * Every argument of both calls is checked before anything is enqueued.
 * q, lens, lens_old, cu_new and the page table must not overlap what the
 * append writes (the cache's codes, metadata and window). */
int kvq_append_decode(const kvq_layout* layout, const kvq_cache* cache,
                      const void* k_new, const void* v_new, int in_dtype,
                      const int32_t* cu_new, const int32_t* lens_old, int max_new,
                      const void* q, int q_dtype, const int32_t* lens, int max_len,
                      float sm_scale, float* out, float* lse,
                      void* workspace, size_t workspace_bytes, kvq_stream_t stream);

/* Bytes of the library's static decode scratch (per device). */
#define KVQ_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* kvq_decode_attention without a caller-supplied workspace.  The pages
 * have no counterpart to this call: it is a deployment convenience.  The
 * split partials live in a file-scope static device array of
 * KVQ_STATIC_SCRATCH_BYTES (16 MiB, 256-byte aligned) that the library
 * holds in each device's context.  Its address is looked up once per
 * device, on that device's first call.  The call allocates and frees
 * nothing.
 * Arguments, output and error behaviour are those of kvq_decode_attention,
 * plus one case: KVQ_ERR_WORKSPACE, with nothing enqueued, when
 * kvq_decode_workspace_bytes(layout, cache->batch, max_len) exceeds
 * KVQ_STATIC_SCRATCH_BYTES.  For scale: the persistent tensor-core kernel
 * needs about 1.3 MB on 148 SMs plus 4 bytes per (sequence, kv-head); the
 * two-phase tcgen05 kernel needs 12 MB for batch 64 at lengths up to 16384
 * with 40/8 heads.
 * The array starts at zero when the library's module is loaded in a
 * device context, which is what the merge tickets inside it need; each call
 * writes every partial before reading it and leaves the tickets at zero.
 * One scratch array serves every call on a device.  Calls whose GPU
 * execution overlaps (different streams without ordering between them, or
 * several host threads) race on it and give undefined results.  Order them
 * on one stream, or use kvq_decode_attention with a workspace per stream.
 * The cached address belongs to the context that was current on the device
 * at the first call: do not call this after cudaDeviceReset, nor from
 * another context on the same device (for example one made current with
 * the driver API), since the address is not looked up again. */
int kvq_decode_attention_static_scratch(const kvq_layout* layout, const kvq_cache* cache,
                                        const void* q, int q_dtype, const int32_t* lens,
                                        int max_len, float sm_scale, float* out, float* lse,
                                        kvq_stream_t stream);

/* Attention of a chunk of new query tokens over the cache (chunked
 * prefill), causal, dequantization fused into the kernel.  The pages give
 * attention for one new query ("Kuantisasi KV cache ...", "Error pada key
 * masuk sebelum softmax": s = qK^T/sqrt(d), a = softmax(s), o = aV) over
 * the stored approximation ("Pertumbuhan cache ..."); a chunk of n queries
 * is read as n such queries under a causal mask.
 * Call kvq_quantize_append with the chunk's keys and values first and
 * advance lens; then sequence b holds lens[b] positions and its
 * n_b = cu_q[b+1] - cu_q[b] queries are its newest n_b positions: query i
 * sits at position lens[b] - n_b + i and attends to positions
 * [0, lens[b] - n_b + i] (pages below lens[b] - W, the bf16 window above;
 * with rotate_keys, page keys are scored with the rotated query).
 * q         device [cu_q[batch]][Hq][d], q_dtype KVQ_BF16 or KVQ_F32
 * cu_q      device int32 [batch+1], non-decreasing, cu_q[0] == 0
 * lens      device int32 [batch], positions including the chunk
 * max_q     host bound: max_q >= every n_b (launch size)
 * sm_scale  score scale (1/sqrt(d) for standard attention)
 * out       device fp32 [cu_q[batch]][Hq][d]; lse device fp32
 *           [cu_q[batch]][Hq] (natural log) or NULL.
 * Sequences with n_b = 0 are skipped.  A sequence with n_b > lens[b] or
 * n_b > max_q is skipped too and its output rows are left untouched.
 * Needs no workspace; allocates nothing. */
int kvq_prefill_attention(const kvq_layout* layout, const kvq_cache* cache,
                          const void* q, int q_dtype, const int32_t* cu_q,
                          const int32_t* lens, int max_q, float sm_scale,
                          float* out, float* lse, kvq_stream_t stream);

/* Reconstruct the cache to fp32 [batch][Hkv][max_len][d] (check path;
 * "dequantization into temporary storage").  Quantized positions give
 * code*scale+zero (keys in the rotated domain when rotate_keys), window
 * positions give their bf16 values; positions >= lens[b] are not written. */
int kvq_dequantize(const kvq_layout* layout, const kvq_cache* cache,
                   const int32_t* lens, int max_len, float* k_out, float* v_out,
                   kvq_stream_t stream);

/* Rotate `rows` key rows [rows][Hkv... flattened][d] exactly as
 * kvq_quantize_append does before quantizing them (check path for the
 * key-only rotation of "Quantize What Counts", Resultaten).
 * k       device [rows][d] (in_dtype KVQ_BF16 or KVQ_F32)
 * out     device fp32 [rows][d] */
int kvq_rotate_keys(const kvq_layout* layout, const void* k, int in_dtype, int rows,
                    float* out, kvq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */

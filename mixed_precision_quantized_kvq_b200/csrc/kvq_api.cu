// C-ABI entry points (declared in include/kvq.h): argument checks on the
// host, launch planning, and dispatch to the kernels.  Nothing is allocated,
// freed or synchronised here.
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "kvq_internal.cuh"
#include "kvq_channel.cuh"
#include "kvq_prefill.cuh"

namespace {

using kvq::Params;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];   // 0 = not queried yet

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < kMaxDevices && g_sm_count[dev] > 0) return g_sm_count[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 148;
    }
    if (dev < kMaxDevices) g_sm_count[dev] = n;
    return n;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool group_ok(int g, int d) { return (g == 16 || g == 32 || g == 64 || g == 128) && g <= d && d % g == 0; }
bool bits_ok(int b) { return b == 1 || b == 2 || b == 4 || b == 8; }

int check_layout(const kvq_layout* l) {
    if (!l) return KVQ_ERR_INVALID_ARG;
    if (l->head_dim != 64 && l->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
    if (l->num_kv_heads <= 0 || l->num_q_heads <= 0) return KVQ_ERR_INVALID_ARG;
    if (l->num_q_heads % l->num_kv_heads) return KVQ_ERR_UNSUPPORTED;
    const int g = l->num_q_heads / l->num_kv_heads;
    if (g > kvq::kMaxGqa) return KVQ_ERR_UNSUPPORTED;
    if (!bits_ok(l->k_bits) || !bits_ok(l->v_bits)) return KVQ_ERR_UNSUPPORTED;
    if (l->k_per_channel != 0 && l->k_per_channel != 1) return KVQ_ERR_INVALID_ARG;
    if (l->k_per_channel) {
        // key groups of 16, 32 or 64 positions of one channel; rotation mixes channels per token
        if (l->k_group != 16 && l->k_group != 32 && l->k_group != 64) return KVQ_ERR_UNSUPPORTED;
        if (l->rotate_keys) return KVQ_ERR_UNSUPPORTED;
    } else if (!group_ok(l->k_group, l->head_dim)) {
        return KVQ_ERR_UNSUPPORTED;
    }
    if (!group_ok(l->v_group, l->head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (l->page_size != kvq::kPage) return KVQ_ERR_UNSUPPORTED;
    if (l->window < 0) return KVQ_ERR_INVALID_ARG;
    if (l->rotate_keys && !l->rot_signs) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

// bf16 ring slots per (sequence, kv-head): the window, plus kg - 1 positions
// of an incomplete key group when key groups run along positions
int ring_slots(const kvq_layout* l) { return l->window + (l->k_per_channel ? l->k_group - 1 : 0); }

int check_cache(const kvq_layout* l, const kvq_cache* c) {
    if (!c) return KVQ_ERR_INVALID_ARG;
    if (c->batch < 0 || c->max_pages_per_seq <= 0 || c->num_pages < 0) return KVQ_ERR_INVALID_ARG;
    if (!c->page_table || !c->k_codes || !c->v_codes || !c->k_meta || !c->v_meta) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(c->k_codes) || !aligned16(c->v_codes) || !aligned16(c->k_meta) || !aligned16(c->v_meta) ||
        !aligned16(c->page_table))
        return KVQ_ERR_INVALID_ARG;
    if (ring_slots(l) > 0) {
        if (!c->k_win || !c->v_win || !aligned16(c->k_win) || !aligned16(c->v_win)) return KVQ_ERR_INVALID_ARG;
    }
    return KVQ_OK;
}

Params make_params(const kvq_layout* l, const kvq_cache* c) {
    Params p{};
    p.d = l->head_dim;
    p.hq = l->num_q_heads;
    p.hkv = l->num_kv_heads;
    p.g = p.hq / p.hkv;
    p.kb = l->k_bits;
    p.vb = l->v_bits;
    p.kg = l->k_group;
    p.vg = l->v_group;
    p.nkg = p.d / p.kg;
    p.nvg = p.d / p.vg;
    p.W = l->window;
    p.rotate = l->rotate_keys ? 1 : 0;
    p.signs = l->rot_signs;
    p.krow_bytes = p.d * p.kb / 8;
    p.vchan_bytes = kvq::kPage * p.vb / 8;
    p.kch = p.krow_bytes < 16 ? p.krow_bytes : 16;
    p.vch = p.vchan_bytes < 16 ? p.vchan_bytes : 16;
    if (c) {
        p.k_codes = static_cast<uint8_t*>(c->k_codes);
        p.v_codes = static_cast<uint8_t*>(c->v_codes);
        p.k_meta = static_cast<uint32_t*>(c->k_meta);
        p.v_meta = static_cast<uint32_t*>(c->v_meta);
        p.k_win = static_cast<__nv_bfloat16*>(c->k_win);
        p.v_win = static_cast<__nv_bfloat16*>(c->v_win);
        p.page_table = c->page_table;
        p.batch = c->batch;
        p.max_pages = c->max_pages_per_seq;
        p.num_pages = c->num_pages;
    }
    return p;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return KVQ_OK;
    cudaGetLastError();   // clear a non-sticky launch error
    return KVQ_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* kvq_status_string(int status) {
    switch (status) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or misaligned buffer)";
        case KVQ_ERR_UNSUPPORTED: return "unsupported configuration (bits, head_dim, group size, page size or GQA ratio)";
        case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
        case KVQ_ERR_CUDA: return "CUDA launch or runtime error";
        default: return "unknown status";
    }
}

int kvq_version(void) { return 200; }

int kvq_page_bytes(const kvq_layout* layout, size_t* k_codes, size_t* k_meta, size_t* v_codes,
                   size_t* v_meta) {
    int rc = check_layout(layout);
    if (rc) return rc;
    const size_t per = size_t(layout->num_kv_heads) * kvq::kPage;
    if (k_codes) *k_codes = per * size_t(layout->head_dim * layout->k_bits / 8);
    if (k_meta)
        *k_meta = layout->k_per_channel
                      ? size_t(layout->num_kv_heads) * (kvq::kPage / layout->k_group) * layout->head_dim * 4
                      : per * size_t(layout->head_dim / layout->k_group) * 4;
    if (v_codes) *v_codes = per * size_t(layout->head_dim * layout->v_bits / 8);
    if (v_meta) *v_meta = per * size_t(layout->head_dim / layout->v_group) * 4;
    return KVQ_OK;
}

int kvq_window_bytes(const kvq_layout* layout, int batch, size_t* bytes) {
    int rc = check_layout(layout);
    if (rc) return rc;
    if (batch < 0 || !bytes) return KVQ_ERR_INVALID_ARG;
    *bytes = size_t(batch) * layout->num_kv_heads * ring_slots(layout) * layout->head_dim * 2;
    return KVQ_OK;
}

size_t kvq_decode_workspace_bytes(const kvq_layout* layout, int batch, int max_len) {
    if (check_layout(layout) || batch < 0 || max_len < 0) return 0;
    Params p = make_params(layout, nullptr);
    if (layout->k_per_channel) {   // partials only when the pairs are split between CTAs
        if (!kvq::decode_pc_supported(p, max_len)) return 0;
        const int splits = kvq::pc_splits(p, batch, max_len, device_sm_count());
        return splits > 1 ? kvq::pc_workspace_bytes(p, batch, splits) : 0;
    }
    kvq::DecodePlan pl = kvq::plan_decode(p, batch, max_len, device_sm_count());
    return kvq::decode_workspace_bytes(p, batch, pl);
}

int kvq_set_decode_path(int path) {
    if (path < 0 || path > 3) return KVQ_ERR_INVALID_ARG;
    kvq::g_decode_path = path;
    return KVQ_OK;
}

int kvq_get_decode_path(const kvq_layout* layout) {
    int rc = check_layout(layout);
    if (rc) return rc;
    Params p = make_params(layout, nullptr);
    if (layout->k_per_channel) return kvq::decode_pc_supported(p, 1) ? 4 : 1;
    const int path = kvq::g_decode_path;
    if (path == 1) return 1;
    if (path == 3) return kvq::tc_supported(p) ? 3 : 1;
    return kvq::mma_supported(p, 1) ? 2 : 1;
}

int kvq_decode_status(unsigned int* wait_timeouts, unsigned int* bad_tickets, int clear) {
    return cuda_status(kvq::decode_status(wait_timeouts, bad_tickets, clear != 0));
}

// decode for key groups along positions: the per-channel decode kernel (its
// pairs split between CTAs when the workspace holds the partials), or the
// chunked-prefill kernel with one query per sequence for the shapes it does not take
static int decode_per_channel(const Params& p, const void* q, int q_dtype, const int32_t* lens, int max_len,
                              float sm_scale, float* out, float* lse, void* ws, size_t ws_bytes,
                              kvq_stream_t stream) {
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (kvq::decode_pc_supported(p, max_len)) {
        int splits = kvq::pc_splits(p, p.batch, max_len, device_sm_count());
        if (splits > 1 && (!ws || ws_bytes < kvq::pc_workspace_bytes(p, p.batch, splits) ||
                           (reinterpret_cast<uintptr_t>(ws) & 255u)))
            splits = 1;   // no room for the partials: one CTA per pair
        return cuda_status(kvq::launch_decode_per_channel(p, q, q_dtype == KVQ_BF16, lens, max_len, sm_scale, out, lse,
                                                          ws, splits, s));
    }
    return cuda_status(kvq::launch_prefill_attention(p, 1, 1, q, q_dtype == KVQ_BF16, nullptr, lens, max_len, 1,
                                                     sm_scale, out, lse, s));
}

int kvq_quantize_append(const kvq_layout* layout, const kvq_cache* cache, const void* k_new,
                        const void* v_new, int in_dtype, const int32_t* cu_new, const int32_t* lens,
                        int max_new, kvq_stream_t stream) {
    int rc = check_layout(layout);
    if (rc) return rc;
    if ((rc = check_cache(layout, cache))) return rc;
    if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (max_new < 0 || !cu_new || !lens) return KVQ_ERR_INVALID_ARG;
    if (max_new > 0 && (!k_new || !v_new)) return KVQ_ERR_INVALID_ARG;
    if (max_new == 0 || cache->batch == 0) return KVQ_OK;
    Params p = make_params(layout, cache);
    if (layout->k_per_channel)
        return cuda_status(kvq::launch_append_per_channel(p, k_new, v_new, in_dtype == KVQ_BF16, cu_new, lens,
                                                          max_new, reinterpret_cast<cudaStream_t>(stream)));
    return cuda_status(kvq::launch_quantize_append(p, k_new, v_new, in_dtype == KVQ_BF16, cu_new, lens, max_new,
                                                   reinterpret_cast<cudaStream_t>(stream)));
}

int kvq_decode_attention(const kvq_layout* layout, const kvq_cache* cache, const void* q, int q_dtype,
                         const int32_t* lens, int max_len, float sm_scale, float* out, float* lse,
                         void* workspace, size_t workspace_bytes, kvq_stream_t stream) {
    int rc = check_layout(layout);
    if (rc) return rc;
    if ((rc = check_cache(layout, cache))) return rc;
    if (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (!q || !lens || !out || max_len < 0 || !isfinite(sm_scale)) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return KVQ_ERR_INVALID_ARG;
    if (cache->batch == 0) return KVQ_OK;
    if (cache->batch > 65535 || layout->num_kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;
    Params p = make_params(layout, cache);
    if (layout->k_per_channel)   // the workspace is optional (used for split pairs when it is large enough)
        return decode_per_channel(p, q, q_dtype, lens, max_len, sm_scale, out, lse, workspace, workspace_bytes,
                                  stream);
    kvq::DecodePlan pl = kvq::plan_decode(p, cache->batch, max_len, device_sm_count());
    const size_t need = kvq::decode_workspace_bytes(p, cache->batch, pl);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return KVQ_ERR_WORKSPACE;
    return cuda_status(kvq::launch_decode(p, q, q_dtype == KVQ_BF16, lens, max_len, sm_scale, out, lse,
                                          workspace, pl, reinterpret_cast<cudaStream_t>(stream)));
}

int kvq_append_decode(const kvq_layout* layout, const kvq_cache* cache, const void* k_new, const void* v_new,
                      int in_dtype, const int32_t* cu_new, const int32_t* lens_old, int max_new, const void* q,
                      int q_dtype, const int32_t* lens, int max_len, float sm_scale, float* out, float* lse,
                      void* workspace, size_t workspace_bytes, kvq_stream_t stream) {
    // the checks of both calls, before anything is enqueued
    int rc = check_layout(layout);
    if (rc) return rc;
    if ((rc = check_cache(layout, cache))) return rc;
    if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (max_new < 0 || !cu_new || !lens_old) return KVQ_ERR_INVALID_ARG;
    if (max_new > 0 && (!k_new || !v_new)) return KVQ_ERR_INVALID_ARG;
    if (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (!q || !lens || !out || max_len < 0 || !isfinite(sm_scale)) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return KVQ_ERR_INVALID_ARG;
    if (cache->batch == 0) return KVQ_OK;
    if (cache->batch > 65535 || layout->num_kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;
    Params p = make_params(layout, cache);
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (layout->k_per_channel) {
        if ((rc = kvq_quantize_append(layout, cache, k_new, v_new, in_dtype, cu_new, lens_old, max_new, stream)))
            return rc;
        return kvq_decode_attention(layout, cache, q, q_dtype, lens, max_len, sm_scale, out, lse, workspace,
                                    workspace_bytes, stream);
    }
    kvq::DecodePlan pl = kvq::plan_decode(p, cache->batch, max_len, device_sm_count());
    const size_t need = kvq::decode_workspace_bytes(p, cache->batch, pl);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return KVQ_ERR_WORKSPACE;
    if (max_new > 0) {
        if ((rc = cuda_status(kvq::launch_quantize_append(p, k_new, v_new, in_dtype == KVQ_BF16, cu_new, lens_old,
                                                          max_new, s))))
            return rc;
        pl.after_append = pl.mma && kvq::append_is_one_launch(p, max_new) ? 1 : 0;
    }
    return cuda_status(kvq::launch_decode(p, q, q_dtype == KVQ_BF16, lens, max_len, sm_scale, out, lse, workspace, pl,
                                          s));
}

int kvq_prefill_attention(const kvq_layout* layout, const kvq_cache* cache, const void* q, int q_dtype,
                          const int32_t* cu_q, const int32_t* lens, int max_q, float sm_scale, float* out,
                          float* lse, kvq_stream_t stream) {
    int rc = check_layout(layout);
    if (rc) return rc;
    if ((rc = check_cache(layout, cache))) return rc;
    if (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (!cu_q || !lens || max_q < 0 || !isfinite(sm_scale)) return KVQ_ERR_INVALID_ARG;
    if (cache->batch > 65535 || layout->num_kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;
    if (max_q == 0 || cache->batch == 0) return KVQ_OK;
    if (!q || !out) return KVQ_ERR_INVALID_ARG;
    Params p = make_params(layout, cache);
    return cuda_status(kvq::launch_prefill_attention(p, layout->k_per_channel, 0, q, q_dtype == KVQ_BF16, cu_q, lens,
                                                     INT32_MAX, max_q, sm_scale, out, lse,
                                                     reinterpret_cast<cudaStream_t>(stream)));
}

int kvq_dequantize(const kvq_layout* layout, const kvq_cache* cache, const int32_t* lens, int max_len,
                   float* k_out, float* v_out, kvq_stream_t stream) {
    int rc = check_layout(layout);
    if (rc) return rc;
    if ((rc = check_cache(layout, cache))) return rc;
    if (!lens || !k_out || !v_out || max_len < 0) return KVQ_ERR_INVALID_ARG;
    if (cache->batch == 0 || max_len == 0) return KVQ_OK;
    Params p = make_params(layout, cache);
    if (layout->k_per_channel)
        return cuda_status(kvq::launch_dequantize_per_channel(p, lens, max_len, k_out, v_out,
                                                              reinterpret_cast<cudaStream_t>(stream)));
    return cuda_status(kvq::launch_dequantize(p, lens, max_len, k_out, v_out,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

int kvq_rotate_keys(const kvq_layout* layout, const void* k, int in_dtype, int rows, float* out,
                    kvq_stream_t stream) {
    int rc = check_layout(layout);
    if (rc) return rc;
    if (!layout->rot_signs) return KVQ_ERR_INVALID_ARG;
    if (in_dtype != KVQ_F32 && in_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (rows < 0 || (rows > 0 && (!k || !out))) return KVQ_ERR_INVALID_ARG;
    if (rows == 0) return KVQ_OK;
    Params p = make_params(layout, nullptr);
    return cuda_status(kvq::launch_rotate_keys(p, k, in_dtype == KVQ_BF16, rows, out,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode with library-held scratch: the split partials go to a static device
// array instead of a caller workspace.  Its address is looked up once per
// device; no allocating call is made.
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[KVQ_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];   // nullptr = not looked up yet on that device

int static_scratch(void** addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
    if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* a = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&a, g_decode_scratch);
        if (e != cudaSuccess || !a) return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
        g_scratch_addr[dev] = a;
    }
    *addr = g_scratch_addr[dev];
    return KVQ_OK;
}

}  // namespace

extern "C" int kvq_decode_attention_static_scratch(const kvq_layout* layout, const kvq_cache* cache,
                                                   const void* q, int q_dtype, const int32_t* lens,
                                                   int max_len, float sm_scale, float* out, float* lse,
                                                   kvq_stream_t stream) {
    int rc = check_layout(layout);
    if (rc) return rc;
    if ((rc = check_cache(layout, cache))) return rc;
    if (q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (!q || !lens || !out || max_len < 0 || !isfinite(sm_scale)) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return KVQ_ERR_INVALID_ARG;
    if (cache->batch == 0) return KVQ_OK;
    if (cache->batch > 65535 || layout->num_kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;
    Params p = make_params(layout, cache);
    if (layout->k_per_channel) {   // the static scratch holds the partials of split pairs when large enough
        void* scratch = nullptr;
        if ((rc = static_scratch(&scratch))) return rc;
        return decode_per_channel(p, q, q_dtype, lens, max_len, sm_scale, out, lse, scratch, KVQ_STATIC_SCRATCH_BYTES,
                                  stream);
    }
    kvq::DecodePlan pl = kvq::plan_decode(p, cache->batch, max_len, device_sm_count());
    if (kvq::decode_workspace_bytes(p, cache->batch, pl) > KVQ_STATIC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((rc = static_scratch(&scratch))) return rc;
    return cuda_status(kvq::launch_decode(p, q, q_dtype == KVQ_BF16, lens, max_len, sm_scale, out, lse, scratch,
                                          pl, reinterpret_cast<cudaStream_t>(stream)));
}

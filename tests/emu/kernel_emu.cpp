// Host emulation of the library's emulatable CUDA kernel bodies, for tests.
//
// usage: kernel_emu <dir>
//   <dir>/params.txt   "name value" lines; "mode" selects the kernel:
//       0  attention (kvq_prefill_body.cuh: chunked prefill, or decode with
//          one_query = 1); writes out.bin, lse.bin
//       1  append with per-channel key groups (kvq_channel_body.cuh: group
//          kernel, then ring kernel); rewrites the cache arrays
//       2  dequantize with per-channel key groups; writes k_out.bin, v_out.bin
//   <dir>/<array>.bin  raw arrays named as in the views
// Built with AddressSanitizer; every array is an exact-size allocation.
#include "emu_ctx.h"

#include "kvq_channel_body.cuh"
#include "kvq_prefill_body.cuh"

#include <climits>

namespace {

int attention(emu::Arrays& A, std::map<std::string, double>& P) {
    using kvq::prefill::View;
    auto I = [&](const char* k, int dflt = 0) { return P.count(k) ? int(P.at(k)) : dflt; };
    View v{};
    v.d = I("d");
    v.hq = I("hq");
    v.hkv = I("hkv");
    v.g = v.hq / v.hkv;
    v.kb = I("kb");
    v.vb = I("vb");
    v.kg = I("kg");
    v.vg = I("vg");
    v.nkg = v.d / v.kg;
    v.nvg = v.d / v.vg;
    v.W = I("W");
    v.rotate = I("rotate");
    v.kpc = I("kpc");
    v.R = v.kpc ? v.W + v.kg - 1 : v.W;
    v.batch = I("batch");
    v.max_pages = I("max_pages");
    v.num_pages = I("num_pages");
    v.krow_bytes = v.d * v.kb / 8;
    v.vchan_bytes = kvq::prefill::kTile * v.vb / 8;
    v.kch = v.krow_bytes < 16 ? v.krow_bytes : 16;
    v.vch = v.vchan_bytes < 16 ? v.vchan_bytes : 16;
    v.kchan_bytes = kvq::prefill::kTile * v.kb / 8;
    v.kchc = v.kchan_bytes < 16 ? v.kchan_bytes : 16;
    v.q_bf16 = I("q_bf16");
    v.one_query = I("one_query");
    v.max_q = I("max_q");
    v.len_cap = I("len_cap", INT_MAX);
    v.scale_log2 = float(P.at("sm_scale")) * 1.4426950408889634f;
    v.signs = A.get<int8_t>("signs");
    v.k_codes = A.get<uint8_t>("k_codes");
    v.v_codes = A.get<uint8_t>("v_codes");
    v.k_meta = A.get<uint32_t>("k_meta");
    v.v_meta = A.get<uint32_t>("v_meta");
    v.k_win = A.get<uint16_t>("k_win");
    v.v_win = A.get<uint16_t>("v_win");
    v.page_table = A.get<int32_t>("page_table");
    v.q = A.get<char>("q");
    v.cu_q = v.one_query ? nullptr : A.get<int32_t>("cu_q");
    v.lens = A.get<int32_t>("lens");
    const int rows = v.one_query ? v.batch : v.cu_q[v.batch];
    v.out = A.make<float>("out", size_t(rows) * v.hq * v.d);
    v.lse = A.make<float>("lse", size_t(rows) * v.hq);
    const int qpc = kvq::prefill::queries_per_cta(v.g);
    emu::run_grid((v.max_q + qpc - 1) / qpc, v.hkv, v.batch, kvq::prefill::kThreads,
                  kvq::prefill::smem_bytes(v.d, v.rotate), [&v](emu::Ctx& cx) {
                      if (v.d == 128)
                          kvq::prefill::body<128>(cx, v);
                      else
                          kvq::prefill::body<64>(cx, v);
                  });
    A.put("out");
    A.put("lse");
    return 0;
}

kvq::chan::View chan_view(emu::Arrays& A, std::map<std::string, double>& P) {
    auto I = [&](const char* k) { return int(P.at(k)); };
    kvq::chan::View v{};
    v.d = I("d");
    v.hkv = I("hkv");
    v.kb = I("kb");
    v.vb = I("vb");
    v.kg = I("kg");
    v.vg = I("vg");
    v.nvg = v.d / v.vg;
    v.W = I("W");
    v.R = v.W + v.kg - 1;
    v.batch = I("batch");
    v.max_pages = I("max_pages");
    v.num_pages = I("num_pages");
    v.kchan_bytes = kvq::chan::kPage * v.kb / 8;
    v.vchan_bytes = kvq::chan::kPage * v.vb / 8;
    v.kch = v.kchan_bytes < 16 ? v.kchan_bytes : 16;
    v.vch = v.vchan_bytes < 16 ? v.vchan_bytes : 16;
    v.k_codes = A.get<uint8_t>("k_codes");
    v.v_codes = A.get<uint8_t>("v_codes");
    v.k_meta = A.get<uint32_t>("k_meta");
    v.v_meta = A.get<uint32_t>("v_meta");
    v.k_win = A.get<uint16_t>("k_win");
    v.v_win = A.get<uint16_t>("v_win");
    v.page_table = A.get<int32_t>("page_table");
    v.lens = A.get<int32_t>("lens");
    return v;
}

int append_pc(emu::Arrays& A, std::map<std::string, double>& P) {
    kvq::chan::View v = chan_view(A, P);
    v.k_new = A.get<char>("k_new");
    v.v_new = A.get<char>("v_new");
    v.in_bf16 = int(P.at("in_bf16"));
    v.cu_new = A.get<int32_t>("cu_new");
    const int max_new = int(P.at("max_new"));
    emu::run_grid((max_new + v.kg - 1) / v.kg, v.hkv, v.batch, kvq::chan::kThreads,
                  kvq::chan::append_smem_bytes(v.d, v.kg, v.nvg),
                  [&v](emu::Ctx& cx) { kvq::chan::append_groups_body(cx, v); });
    emu::run_grid(v.hkv, v.batch, 1, kvq::chan::kThreads, 0,
                  [&v](emu::Ctx& cx) { kvq::chan::ring_write_body(cx, v); });
    for (const char* n : {"k_codes", "v_codes", "k_meta", "v_meta", "k_win", "v_win"}) A.put(n);
    return 0;
}

int dequant_pc(emu::Arrays& A, std::map<std::string, double>& P) {
    kvq::chan::View v = chan_view(A, P);
    v.max_len = int(P.at("max_len"));
    const size_t n = size_t(v.batch) * v.hkv * v.max_len * v.d;
    v.k_out = A.make<float>("k_out", n);
    v.v_out = A.make<float>("v_out", n);
    emu::run_grid((v.max_len + kvq::chan::kPage - 1) / kvq::chan::kPage, v.hkv, v.batch, kvq::chan::kThreads, 0,
                  [&v](emu::Ctx& cx) { kvq::chan::dequant_body(cx, v); });
    A.put("k_out");
    A.put("v_out");
    return 0;
}

}  // namespace

int main(int argc, char** argv) {
    if (argc != 2) {
        std::fprintf(stderr, "usage: %s <dir>\n", argv[0]);
        return 2;
    }
    emu::Arrays A(argv[1]);
    auto P = emu::read_params(argv[1]);
    switch (int(P.at("mode"))) {
        case 0: return attention(A, P);
        case 1: return append_pc(A, P);
        case 2: return dequant_pc(A, P);
        default: return 2;
    }
}

// Host emulation of the chunked-prefill attention kernel, for tests only.
//
// Runs the kernel's own per-CTA body (kvq_prefill_body.cuh) on the CPU: one
// std::thread per CUDA thread, std::barrier for __syncthreads, and warp
// reductions that take the same butterfly steps as the shuffles on the GPU.
// Every input array is its own exact-size heap allocation and the program
// is built with AddressSanitizer, so an out-of-range index in the kernel
// body fails the run.  Blocks run one after another.
//
// usage: prefill_emu <dir>
//   <dir>/params.txt   "name value" lines (layout, cache and call scalars)
//   <dir>/<array>.bin  raw arrays named as in prefill::View
// writes <dir>/out.bin (fp32 [total_q][Hq][d]) and <dir>/lse.bin.
#include <cuda_runtime.h>

#include <barrier>
#include <cstdio>
#include <cstdlib>
#include <fstream>
#include <map>
#include <memory>
#include <sstream>
#include <string>
#include <thread>
#include <vector>

#include "kvq_prefill_body.cuh"

using kvq::prefill::View;
constexpr int NT = kvq::prefill::kThreads;

namespace {

struct Block {
    int bx, by, bz;
    float* smem;
    std::barrier<> block_bar{NT};
    std::vector<std::unique_ptr<std::barrier<>>> warp_bar;
    float warp_buf[NT];
    Block() {
        for (int w = 0; w < NT / 32; ++w) warp_bar.emplace_back(new std::barrier<>(32));
    }
};

struct HostCtx {
    Block* blk;
    int t;
    int tid() const { return t; }
    int bx() const { return blk->bx; }
    int by() const { return blk->by; }
    int bz() const { return blk->bz; }
    float* smem() const { return blk->smem; }
    void sync() const { blk->block_bar.arrive_and_wait(); }
    template <class Op>
    float butterfly(float x, Op op) const {
        const int w = t / 32, lane = t % 32;
        blk->warp_buf[t] = x;
        blk->warp_bar[w]->arrive_and_wait();
        float v[32];
        for (int l = 0; l < 32; ++l) v[l] = blk->warp_buf[w * 32 + l];
        blk->warp_bar[w]->arrive_and_wait();
        for (int m = 16; m; m >>= 1) {
            float nv[32];
            for (int l = 0; l < 32; ++l) nv[l] = op(v[l], v[l ^ m]);
            for (int l = 0; l < 32; ++l) v[l] = nv[l];
        }
        return v[lane];
    }
    float warp_max(float x) const { return butterfly(x, [](float a, float b) { return fmaxf(a, b); }); }
    float warp_sum(float x) const { return butterfly(x, [](float a, float b) { return a + b; }); }
};

template <class T>
T* load(const std::string& dir, const std::string& name, std::vector<void*>& owned) {
    std::ifstream f(dir + "/" + name + ".bin", std::ios::binary | std::ios::ate);
    if (!f) return nullptr;
    const size_t n = size_t(f.tellg());
    f.seekg(0);
    char* p = new char[n > 0 ? n : 1];
    f.read(p, std::streamsize(n));
    owned.push_back(p);
    return reinterpret_cast<T*>(p);
}

}  // namespace

int main(int argc, char** argv) {
    if (argc != 2) {
        fprintf(stderr, "usage: %s <dir>\n", argv[0]);
        return 2;
    }
    const std::string dir = argv[1];
    std::map<std::string, double> P;
    {
        std::ifstream f(dir + "/params.txt");
        std::string k;
        double v;
        while (f >> k >> v) P[k] = v;
    }
    auto I = [&](const char* k) { return int(P.at(k)); };
    std::vector<void*> owned;
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
    v.batch = I("batch");
    v.max_pages = I("max_pages");
    v.num_pages = I("num_pages");
    v.krow_bytes = v.d * v.kb / 8;
    v.vchan_bytes = kvq::prefill::kTile * v.vb / 8;
    v.kch = v.krow_bytes < 16 ? v.krow_bytes : 16;
    v.vch = v.vchan_bytes < 16 ? v.vchan_bytes : 16;
    v.q_bf16 = I("q_bf16");
    v.max_q = I("max_q");
    v.scale_log2 = float(P.at("sm_scale")) * 1.4426950408889634f;
    v.signs = load<int8_t>(dir, "signs", owned);
    v.k_codes = load<uint8_t>(dir, "k_codes", owned);
    v.v_codes = load<uint8_t>(dir, "v_codes", owned);
    v.k_meta = load<uint32_t>(dir, "k_meta", owned);
    v.v_meta = load<uint32_t>(dir, "v_meta", owned);
    v.k_win = load<uint16_t>(dir, "k_win", owned);
    v.v_win = load<uint16_t>(dir, "v_win", owned);
    v.page_table = load<int32_t>(dir, "page_table", owned);
    v.q = load<char>(dir, "q", owned);
    v.cu_q = load<int32_t>(dir, "cu_q", owned);
    v.lens = load<int32_t>(dir, "lens", owned);
    const int total_q = v.cu_q[v.batch];
    std::vector<float> out(size_t(total_q) * v.hq * v.d, 0.f), lse(size_t(total_q) * v.hq, 0.f);
    // exact-size output buffers so that ASan sees writes past the end
    float* out_p = new float[out.size() > 0 ? out.size() : 1]();
    float* lse_p = new float[lse.size() > 0 ? lse.size() : 1]();
    v.out = out_p;
    v.lse = lse_p;

    const int qpc = kvq::prefill::queries_per_cta(v.g);
    const int gx = (v.max_q + qpc - 1) / qpc;
    const size_t sm = kvq::prefill::smem_bytes(v.d, v.rotate);
    for (int bz = 0; bz < v.batch; ++bz)
        for (int by = 0; by < v.hkv; ++by)
            for (int bx = 0; bx < gx; ++bx) {
                Block blk;
                blk.bx = bx;
                blk.by = by;
                blk.bz = bz;
                std::unique_ptr<char[]> s(new char[sm]);
                blk.smem = reinterpret_cast<float*>(s.get());
                std::vector<std::thread> th;
                for (int t = 0; t < NT; ++t)
                    th.emplace_back([&blk, t, &v] {
                        HostCtx cx{&blk, t};
                        if (v.d == 128)
                            kvq::prefill::body<128>(cx, v);
                        else
                            kvq::prefill::body<64>(cx, v);
                    });
                for (auto& x : th) x.join();
            }
    std::ofstream(dir + "/out.bin", std::ios::binary)
        .write(reinterpret_cast<const char*>(out_p), std::streamsize(out.size() * 4));
    std::ofstream(dir + "/lse.bin", std::ios::binary)
        .write(reinterpret_cast<const char*>(lse_p), std::streamsize(lse.size() * 4));
    delete[] out_p;
    delete[] lse_p;
    for (void* p : owned) delete[] static_cast<char*>(p);
    return 0;
}

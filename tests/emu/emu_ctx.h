// Host execution of a CUDA kernel body, for tests only: one std::thread per
// CUDA thread, std::barrier for __syncthreads, warp reductions that take the
// GPU's butterfly steps, the IEEE fp32 operations with directed rounding
// through the C library's rounding modes, fp16/bf16 conversions through the
// CUDA headers' host functions, and 32-bit atomics through
// std::atomic_ref.  Blocks run one after another.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <barrier>
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <fstream>
#include <map>
#include <memory>
#include <string>
#include <thread>
#include <vector>

namespace emu {

struct Block {
    int nt;
    int bx = 0, by = 0, bz = 0;
    float* smem = nullptr;
    std::barrier<> block_bar;
    std::vector<std::unique_ptr<std::barrier<>>> warp_bar;
    std::vector<float> warp_buf;
    explicit Block(int threads) : nt(threads), block_bar(threads), warp_buf(threads) {
        for (int w = 0; w < threads / 32; ++w) warp_bar.emplace_back(new std::barrier<>(32));
    }
};

// fp32 a op b rounded toward +inf (op 0: subtract, 1: divide)
inline float op_up(float a, float b, int op) {
    const int old = std::fegetround();
    std::fesetround(FE_UPWARD);
    volatile float va = a, vb = b;
    volatile float r = op == 0 ? va - vb : va / vb;
    std::fesetround(old);
    return r;
}

struct Ctx {
    Block* blk;
    int t;
    int tid() const { return t; }
    int nthreads() const { return blk->nt; }
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
    float warp_max(float x) const { return butterfly(x, [](float a, float b) { return std::fmax(a, b); }); }
    float warp_sum(float x) const { return butterfly(x, [](float a, float b) { return a + b; }); }
    uint16_t f2h_rd(float x) const { return __half_as_ushort(__float2half_rd(x)); }
    uint16_t f2h_ru(float x) const { return __half_as_ushort(__float2half_ru(x)); }
    float sub_ru(float a, float b) const { return op_up(a, b, 0); }
    float div_ru(float a, float b) const { return op_up(a, b, 1); }
    float sub_rn(float a, float b) const {
        volatile float va = a, vb = b;
        return va - vb;
    }
    float div_rn(float a, float b) const {
        volatile float va = a, vb = b;
        return va / vb;
    }
    float mul_rn(float a, float b) const {
        volatile float va = a, vb = b;
        return va * vb;
    }
    uint16_t f2bf_rn(float x) const { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
    void atomic_and(uint32_t* p, uint32_t v) const { std::atomic_ref<uint32_t>(*p).fetch_and(v); }
    void atomic_or(uint32_t* p, uint32_t v) const { std::atomic_ref<uint32_t>(*p).fetch_or(v); }
};

// Run body(ctx) for every block of grid (gx, gy, gz) with nt threads and
// smem_bytes of shared memory (an exact-size heap block).
template <class F>
void run_grid(int gx, int gy, int gz, int nt, size_t smem_bytes, F body) {
    for (int z = 0; z < gz; ++z)
        for (int y = 0; y < gy; ++y)
            for (int x = 0; x < gx; ++x) {
                Block blk(nt);
                blk.bx = x;
                blk.by = y;
                blk.bz = z;
                std::unique_ptr<char[]> s(smem_bytes ? new char[smem_bytes] : nullptr);
                blk.smem = reinterpret_cast<float*>(s.get());
                std::vector<std::thread> th;
                for (int t = 0; t < nt; ++t)
                    th.emplace_back([&blk, t, &body] {
                        Ctx cx{&blk, t};
                        body(cx);
                    });
                for (auto& x : th) x.join();
            }
}

// "name value" lines
inline std::map<std::string, double> read_params(const std::string& dir) {
    std::map<std::string, double> P;
    std::ifstream f(dir + "/params.txt");
    std::string k;
    double v;
    while (f >> k >> v) P[k] = v;
    return P;
}

// Arrays read from <dir>/<name>.bin into exact-size heap blocks (so that
// AddressSanitizer sees any access past their end); written back on demand.
struct Arrays {
    std::string dir;
    std::map<std::string, std::pair<char*, size_t>> a;
    explicit Arrays(std::string d) : dir(std::move(d)) {}
    ~Arrays() {
        for (auto& kv : a) delete[] kv.second.first;
    }
    template <class T>
    T* get(const std::string& name) {
        std::ifstream f(dir + "/" + name + ".bin", std::ios::binary | std::ios::ate);
        if (!f) return nullptr;
        const size_t n = size_t(f.tellg());
        f.seekg(0);
        char* p = new char[n > 0 ? n : 1];
        f.read(p, std::streamsize(n));
        a[name] = {p, n};
        return reinterpret_cast<T*>(p);
    }
    template <class T>
    T* make(const std::string& name, size_t count) {
        char* p = new char[count * sizeof(T) > 0 ? count * sizeof(T) : 1]();
        a[name] = {p, count * sizeof(T)};
        return reinterpret_cast<T*>(p);
    }
    void put(const std::string& name) {
        auto& e = a.at(name);
        std::ofstream(dir + "/" + name + ".bin", std::ios::binary).write(e.first, std::streamsize(e.second));
    }
};

}  // namespace emu

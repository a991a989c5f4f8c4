// The oracle's fp32 -> fp16 conversion (kvqo_f32_to_f16: nearest-even,
// toward -inf, toward +inf) against the CUDA headers' host implementations
// of __float2half_rn / _rd / _ru, and its fp32 -> bf16 nearest-even
// conversion (kvqo_f32_to_bf16) against __float2bfloat16_rn; for tests only.
//
// usage: f16_crosscheck <liboracle.so> <stride>
// Checks every fp32 bit pattern whose magnitude lies in [2^-25, 2^17)
// (every pattern that rounds to a nonzero finite fp16 or to the overflow
// boundary, both signs), plus every stride-th pattern of all 2^32 (zeros,
// subnormals, huge values, infinities, NaNs: NaN only has to stay NaN),
// and every stride-th pattern through the bf16 conversion.
// Prints "<checked> <mismatches>" and exits non-zero on a mismatch.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <dlfcn.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>

typedef uint16_t (*conv_t)(float, int);

static bool is_nan16(uint16_t h) { return (h & 0x7c00u) == 0x7c00u && (h & 0x03ffu); }
static bool is_nan_bf16(uint16_t h) { return (h & 0x7f80u) == 0x7f80u && (h & 0x007fu); }

static long long check(conv_t f, uint32_t u) {
    float x;
    std::memcpy(&x, &u, 4);
    long long bad = 0;
    for (int mode = -1; mode <= 1; ++mode) {
        const uint16_t a = f(x, mode);
        const __half hb = mode < 0 ? __float2half_rd(x) : mode > 0 ? __float2half_ru(x) : __float2half_rn(x);
        const uint16_t b = __half_as_ushort(hb);
        if (std::isnan(x)) bad += !(is_nan16(a) && is_nan16(b));
        else bad += a != b;
    }
    return bad;
}

int main(int argc, char** argv) {
    if (argc != 3) return 2;
    void* h = dlopen(argv[1], RTLD_NOW);
    if (!h) return 2;
    conv_t f = reinterpret_cast<conv_t>(dlsym(h, "kvqo_f32_to_f16"));
    conv_t fb = reinterpret_cast<conv_t>(dlsym(h, "kvqo_f32_to_bf16"));
    if (!f || !fb) return 2;
    const long long stride = std::atoll(argv[2]);
    const uint32_t lo = 0x33000000u, hi = 0x48000000u;   // |x| in [2^-25, 2^17)
    long long bad = 0, n = 0;
#pragma omp parallel for reduction(+ : bad, n) schedule(static)
    for (long long i = lo; i < (long long)hi; ++i) {
        bad += check(f, uint32_t(i)) + check(f, uint32_t(i) | 0x80000000u);
        n += 6;
    }
#pragma omp parallel for reduction(+ : bad, n) schedule(static)
    for (long long i = 0; i < (1LL << 32); i += stride) {
        bad += check(f, uint32_t(i));
        n += 3;
    }
#pragma omp parallel for reduction(+ : bad, n) schedule(static)
    for (long long i = 0; i < (1LL << 32); i += stride / 8 > 0 ? stride / 8 : 1) {
        const uint32_t u = uint32_t(i);
        float x;
        std::memcpy(&x, &u, 4);
        const uint16_t a = fb(x, 0), b = __bfloat16_as_ushort(__float2bfloat16_rn(x));
        bad += std::isnan(x) ? !(is_nan_bf16(a) && is_nan_bf16(b)) : a != b;
        n += 1;
    }
    std::printf("%lld %lld\n", n, bad);
    return bad != 0;
}

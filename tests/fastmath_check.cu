// Checks of the step kernel's fast square root and division (fastmath.cuh)
// against CUDA's correctly rounded __fsqrt_rn and __fdiv_rn:
//   sqrt:  every float in [2^-100, FLT_MAX] (the range sqrt_fast_ok accepts);
//   rcp:   every float d in [2^-60, 2^64] gives 1/d rounded to nearest;
//   div:   random pairs over the whole range of div2_fast (dividends of
//          both signs, divisors with random, all-ones and near-all-ones
//          significands), and every dividend significand in four binades
//          against 4096 divisors just below a power of two;
//   dequant_steps / quant_factors: every 32-bit pattern (both signs,
//          zeros, subnormals, infinities, NaNs) against their definitions
//          x/127, x/255 and (x > 0 ? 127/x : 0), (x > 0 ? 255/x : 0).
// Prints one line per check; built and run by tests/test_gpu_fastmath.py.
#include <cstdio>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "fastmath.cuh"

using namespace dbuf_k;

struct Tally {
    unsigned long long checked, bad;
    uint32_t example;
};

__device__ void tally(Tally* t, unsigned long long n, unsigned long long b, uint32_t ex) {
    if (n) atomicAdd(&t->checked, n);
    if (b) {
        atomicAdd(&t->bad, b);
        t->example = ex;
    }
}

__device__ __forceinline__ bool differ(float a, float b) { return __float_as_uint(a) != __float_as_uint(b); }

__global__ void check_sqrt(Tally* t, uint32_t first_pair, uint32_t end_bits) {
    const uint32_t i = first_pair + blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t u0 = 2u * i, u1 = 2u * i + 1u;
    if (u0 >= end_bits) return;
    const uint32_t w1 = u1 < end_bits ? u1 : u0;
    const float2 v = make_float2(__uint_as_float(u0), __uint_as_float(w1));
    if (!sqrt_fast_ok(v.x) || !sqrt_fast_ok(v.y)) return;
    const float2 r = sqrt2_fast(v);
    const bool b0 = differ(r.x, __fsqrt_rn(v.x)), b1 = differ(r.y, __fsqrt_rn(v.y));
    tally(t, 2, b0 + b1, b0 ? u0 : w1);
}

// Every d in [lo_bits, hi_bits], two per thread.
__global__ void check_rcp(Tally* t, uint32_t first_pair, uint32_t lo_bits, uint32_t hi_bits) {
    const uint32_t i = first_pair + blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t u0 = 2u * i, u1 = 2u * i + 1u;
    if (u0 > hi_bits || u1 < lo_bits) return;
    const uint32_t a = u0 < lo_bits ? lo_bits : u0, b = u1 > hi_bits ? hi_bits : u1;
    const float2 d = make_float2(__uint_as_float(a), __uint_as_float(b));
    const float2 y = rcp2_fast(d);
    const bool b0 = differ(y.x, __fdiv_rn(1.f, d.x)), b1 = differ(y.y, __fdiv_rn(1.f, d.y));
    tally(t, 2, b0 + b1, b0 ? a : b);
}

__device__ __forceinline__ uint64_t splitmix(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Random (a, d): exponents uniform over the accepted ranges, significands
// random; one in four divisors has an all-ones significand, one in eight is
// within 8 ulps below a power of two.
__global__ void check_div_random(Tally* t, uint64_t base) {
    const uint64_t i = base + blockIdx.x * (uint64_t)blockDim.x + threadIdx.x;
    const uint64_t h = splitmix(i), h2 = splitmix(i ^ 0x5555555555555555ull);
    float2 a, d;
    for (int k = 0; k < 2; ++k) {
        const uint64_t g = k ? h2 : h;
        const uint32_t ea = 127u - 61u + (uint32_t)((g >> 40) % 129u);   // [2^-61, 2^68)
        const uint32_t ed = 127u - 60u + (uint32_t)((g >> 50) % 124u);   // [2^-60, 2^64)
        uint32_t sd = (uint32_t)(g >> 23) & 0x7FFFFFu;
        if ((i & 3) == 1) sd = 0x7FFFFFu;
        if ((i & 7) == 2) sd = 0x7FFFFFu - (uint32_t)((g >> 60) & 7u);
        const float av = __uint_as_float((ea << 23) | ((uint32_t)g & 0x7FFFFFu) | ((g >> 63) ? 0x80000000u : 0u));
        const float dv = __uint_as_float((ed << 23) | sd);
        if (k) { a.y = av; d.y = dv; } else { a.x = av; d.x = dv; }
    }
    const float2 q = div2_fast(a, d);
    const bool b0 = differ(q.x, __fdiv_rn(a.x, d.x)), b1 = differ(q.y, __fdiv_rn(a.y, d.y));
    tally(t, 2, b0 + b1, b0 ? __float_as_uint(d.x) : __float_as_uint(d.y));
}

// Every dividend significand in binades 2^0, 2^7, 2^14, 2^21 against the
// divisor 2 - (sel + 1) ulp.
__global__ void check_div_grid(Tally* t, uint32_t sel) {
    const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;     // 2^24 threads, 2 quotients each
    const uint32_t s = (i & 0x3FFFFFu) << 1, ex = i >> 22;
    const float2 a = make_float2(__uint_as_float(((127u + 7u * ex) << 23) | s),
                                 __uint_as_float(((127u + 7u * ex) << 23) | (s + 1u)));
    const float dv = __uint_as_float((127u << 23) | (0x7FFFFFu - sel));
    const float2 q = div2_fast(a, make_float2(dv, dv));
    const bool b0 = differ(q.x, __fdiv_rn(a.x, dv)), b1 = differ(q.y, __fdiv_rn(a.y, dv));
    tally(t, 2, b0 + b1, __float_as_uint(dv));
}

static uint32_t bits_of(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return u;
}

// Every bit pattern u in [first, first + n), one per thread.
__global__ void check_factors(Tally* t, uint64_t first) {
    const uint64_t i = first + blockIdx.x * (uint64_t)blockDim.x + threadIdx.x;
    if (i > 0xFFFFFFFFull) return;
    const float x = __uint_as_float((uint32_t)i);
    const float2 dq = dequant_steps(make_float2(x, x));
    const bool b0 = differ(dq.x, __fdiv_rn(x, 127.f)) || differ(dq.y, __fdiv_rn(x, 255.f));
    const float2 qf = quant_factors(make_float2(x, x));
    const bool b1 = differ(qf.x, x > 0.f ? __fdiv_rn(127.f, x) : 0.f) || differ(qf.y, x > 0.f ? __fdiv_rn(255.f, x) : 0.f);
    tally(t, 2, b0 + b1, (uint32_t)i);
}

int main() {
    Tally* t;
    if (cudaMalloc(&t, 5 * sizeof(Tally)) != cudaSuccess) return 2;
    cudaMemset(t, 0, 5 * sizeof(Tally));
    {   // sqrt: [2^-100, +inf)
        const uint32_t lo = kSqrtFastMinBits, hi = 0x7F800000u, per = 1u << 26;
        for (uint32_t p = lo / 2u; p < hi / 2u; p += per) {
            const uint32_t n = hi / 2u - p < per ? hi / 2u - p : per;
            check_sqrt<<<(n + 255) / 256, 256>>>(t + 0, p, hi);
        }
    }
    {   // rcp: [2^-60, 2^64]
        const uint32_t lo = bits_of(kDivMinD), hi = bits_of(kDivMaxD), per = 1u << 26;
        for (uint32_t p = lo / 2u; p <= hi / 2u; p += per) {
            const uint32_t n = hi / 2u + 1u - p < per ? hi / 2u + 1u - p : per;
            check_rcp<<<(n + 255) / 256, 256>>>(t + 1, p, lo, hi);
        }
    }
    for (uint64_t b = 0; b < (1ull << 33); b += (1ull << 27))       // 2^34 random quotients
        check_div_random<<<(1u << 27) / 256, 256>>>(t + 2, b);
    for (uint32_t sel = 0; sel < 4096; ++sel)                       // 2^37 structured quotients
        check_div_grid<<<(1u << 24) / 256, 256>>>(t + 3, sel);
    for (uint64_t b = 0; b < (1ull << 32); b += (1ull << 28))       // every 32-bit pattern
        check_factors<<<(1u << 28) / 256, 256>>>(t + 4, b);
    Tally h[5];
    const cudaError_t err = cudaMemcpy(h, t, sizeof h, cudaMemcpyDeviceToHost);
    const char* names[5] = {"sqrt", "rcp", "div_random", "div_grid", "block_factors"};
    for (int k = 0; k < 5; ++k)
        printf("%s checked=%llu mismatches=%llu example=%08x\n", names[k], h[k].checked, h[k].bad, h[k].example);
    printf("status=%s\n", cudaGetErrorString(err));
    return err == cudaSuccess ? 0 : 1;
}

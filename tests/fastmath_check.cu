// Exhaustive check of the step kernel's square root (fastmath.cuh) against
// CUDA's correctly rounded __fsqrt_rn: every float bit pattern in
// [2^-100, FLT_MAX] (the range sqrt_fast_ok accepts).  Prints the number of
// differing results; built and run by tests/test_gpu_fastmath.py.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>

#include "fastmath.cuh"

__global__ void check(unsigned long long* bad, uint32_t* example, uint32_t first_pair, uint32_t end_bits) {
    const uint32_t i = first_pair + blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t u0 = 2u * i, u1 = 2u * i + 1u;
    if (u0 >= end_bits) return;
    const uint32_t w1 = u1 < end_bits ? u1 : u0;
    const float2 v = make_float2(__uint_as_float(u0), __uint_as_float(w1));
    if (!dbuf_k::sqrt_fast_ok(v.x) || !dbuf_k::sqrt_fast_ok(v.y)) return;
    const float2 r = dbuf_k::sqrt2_fast(v);
    const bool b0 = __float_as_uint(r.x) != __float_as_uint(__fsqrt_rn(v.x));
    const bool b1 = __float_as_uint(r.y) != __float_as_uint(__fsqrt_rn(v.y));
    if (b0 || b1) {
        atomicAdd(bad, 1ull);
        *example = b0 ? u0 : w1;
    }
}

int main() {
    const uint32_t lo = dbuf_k::kSqrtFastMinBits, hi = 0x7F800000u;  // [2^-100, +inf)
    unsigned long long* bad;
    uint32_t* ex;
    if (cudaMalloc(&bad, 8) != cudaSuccess || cudaMalloc(&ex, 4) != cudaSuccess) return 2;
    cudaMemset(bad, 0, 8);
    cudaMemset(ex, 0, 4);
    const uint32_t first = lo / 2u, last = hi / 2u, per = 1u << 26;
    for (uint32_t p = first; p < last; p += per) {
        const uint32_t n = last - p < per ? last - p : per;
        check<<<(n + 255) / 256, 256>>>(bad, ex, p, hi);
    }
    unsigned long long h = 0;
    uint32_t e = 0;
    const cudaError_t err = cudaMemcpy(&h, bad, 8, cudaMemcpyDeviceToHost);
    cudaMemcpy(&e, ex, 4, cudaMemcpyDeviceToHost);
    printf("checked=%u mismatches=%llu example=%08x status=%s\n", hi - lo, h, e, cudaGetErrorString(err));
    return err == cudaSuccess ? 0 : 1;
}

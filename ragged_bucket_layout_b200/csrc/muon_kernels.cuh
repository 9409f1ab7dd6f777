// Element-wise kernels of the Muon step (the matrix products of the
// Newton-Schulz iteration run as cuBLAS GEMMs): momentum with the direction
// and its squared norm, the normalised bf16 start, and the weight update.
// Sums are fp64 per thread, per-CTA partials in a fixed order, so results do
// not depend on scheduling.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace dbuf_k {

constexpr int kMuonThreads = 256;
constexpr int kMuonMaxCTAs = 1024;

__device__ __forceinline__ float bf16_to_float(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

__device__ __forceinline__ void block_sum_to(double acc, double* out) {
    __shared__ double part[kMuonThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_down_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int w = 0; w < kMuonThreads / 32; ++w) s += part[w];
        *out = s;
    }
}

// t = g * gs; mom = beta * mom + t; u = t + beta * mom (nesterov) or mom;
// partial[cta] = sum of u^2 over the CTA's elements (fp64).
__global__ void __launch_bounds__(kMuonThreads) muon_momentum_kernel(const uint16_t* __restrict__ g,
                                                                    float* __restrict__ mom, float* __restrict__ u,
                                                                    int64_t n, float beta, float gs, int nesterov,
                                                                    double* __restrict__ partial) {
    double acc = 0.0;
    for (int64_t i = blockIdx.x * (int64_t)kMuonThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kMuonThreads) {
        const float t = __fmul_rn(bf16_to_float(g[i]), gs);
        const float m = __fadd_rn(__fmul_rn(beta, mom[i]), t);
        mom[i] = m;
        const float d = nesterov ? __fadd_rn(t, __fmul_rn(beta, m)) : m;
        u[i] = d;
        acc += (double)d * (double)d;
    }
    block_sum_to(acc, partial + blockIdx.x);
}

// partial[cta] = sum of u^2 over the CTA's elements.
__global__ void __launch_bounds__(kMuonThreads) muon_sumsq_kernel(const float* __restrict__ u, int64_t n,
                                                                 double* __restrict__ partial) {
    double acc = 0.0;
    for (int64_t i = blockIdx.x * (int64_t)kMuonThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kMuonThreads)
        acc += (double)u[i] * (double)u[i];
    block_sum_to(acc, partial + blockIdx.x);
}

// x = bf16(u / (sqrt(sum of partials) + eps)); every CTA adds the partials
// itself, in index order.
__global__ void __launch_bounds__(kMuonThreads) muon_normalise_kernel(const float* __restrict__ u, int64_t n,
                                                                     const double* __restrict__ partial, int n_part,
                                                                     float eps, __nv_bfloat16* __restrict__ x) {
    __shared__ float inv;
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int j = 0; j < n_part; ++j) s += partial[j];
        inv = (float)(1.0 / (sqrt(s) + (double)eps));
    }
    __syncthreads();
    const float f = inv;
    for (int64_t i = blockIdx.x * (int64_t)kMuonThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kMuonThreads)
        x[i] = __float2bfloat16_rn(__fmul_rn(u[i], f));
}

// master = master * decay - lrs * x;  param = bf16(master).
__global__ void __launch_bounds__(kMuonThreads) muon_update_kernel(float* __restrict__ master,
                                                                  uint16_t* __restrict__ param,
                                                                  const __nv_bfloat16* __restrict__ x, int64_t n,
                                                                  float decay, float lrs) {
    for (int64_t i = blockIdx.x * (int64_t)kMuonThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kMuonThreads) {
        const float p = __fsub_rn(__fmul_rn(master[i], decay), __fmul_rn(lrs, __bfloat162float(x[i])));
        master[i] = p;
        param[i] = __bfloat16_as_ushort(__float2bfloat16_rn(p));
    }
}

}  // namespace dbuf_k

// DBuffer group operations beyond scale and zero (veScale-FSDP paper Sec. 5,
// gist.science "Technische samenvatting" 2C: identical operations such as
// add, scale and zero are fused across the tensors of a bucket):
//   * gradient accumulation across micro-batches (group add) shares the
//     copy-in kernel of pack_kernel.cuh (the accumulate instance);
//   * global L2 norm of the scaled gradient bucket, and the clipping factor
//     folded into the step's grad_scale on the device.
//
// The norm is deterministic: every thread sums its squares in double in a
// fixed order, each CTA writes its partial sum to scratch memory, and the
// last CTA to finish adds the partials in a fixed order.
#pragma once

#include <cuda_bf16.h>

#include "tma.cuh"

namespace dbuf_k {

constexpr int kNormThreads = 256;
constexpr int kNormMaxCTAs = 2048;

// Scratch of the norm reduction (global memory, zero at first use; the last
// CTA puts the counter back to zero).
struct NormScratch {
    double partial[kNormMaxCTAs];
    uint32_t counter;
    uint32_t pad_;
    double norm;
    float gscale_eff;  // grad_scale after clipping, read by the step kernel
    float pad2_;
};

__device__ __forceinline__ double block_sum_fixed(double v, double* s_warp) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v += __shfl_down_sync(0xffffffffu, v, d);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) s_warp[warp] = v;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < kNormThreads / 32; ++w) t += s_warp[w];
    return t;  // valid in thread 0
}

// Sum of squares of float(grad[i]) * grad_scale (the step's scaled
// gradient), i < n, in double; the last CTA writes sqrt(sum) and the
// clipped scale.  clip = 0: gscale_eff = grad_scale.
__global__ void __launch_bounds__(kNormThreads)
    grad_norm_kernel(const uint16_t* __restrict__ grad, int64_t n, float grad_scale, float max_norm, int clip,
                     NormScratch* sc, double* norm_out) {
    __shared__ double s_warp[kNormThreads / 32];
    __shared__ int s_last;
    double acc = 0.0;
    const int64_t nv = n / 8;
    const int64_t stride = (int64_t)gridDim.x * kNormThreads;
    for (int64_t v = (int64_t)blockIdx.x * kNormThreads + threadIdx.x; v < nv; v += stride) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(grad) + v);
        const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double a = (double)__fmul_rn(__uint_as_float(q[i] << 16), grad_scale);
            const double b = (double)__fmul_rn(__uint_as_float(q[i] & 0xffff0000u), grad_scale);
            acc = __fma_rn(a, a, acc);  // a*a is exact in double
            acc = __fma_rn(b, b, acc);
        }
    }
    if (blockIdx.x == 0 && threadIdx.x < (int)(n - nv * 8)) {  // tail of fewer than 8 elements
        const double a = (double)__fmul_rn(__uint_as_float((uint32_t)grad[nv * 8 + threadIdx.x] << 16), grad_scale);
        acc = __fma_rn(a, a, acc);
    }
    const double part = block_sum_fixed(acc, s_warp);
    if (threadIdx.x == 0) {
        sc->partial[blockIdx.x] = part;
        __threadfence();
        const uint32_t prev = atomicAdd(&sc->counter, 1u);
        s_last = (prev == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    if (!s_last) return;
    // Last CTA: add the partials in a fixed order.
    __threadfence();
    double t = 0.0;
    for (int i = threadIdx.x; i < (int)gridDim.x; i += kNormThreads)
        t += *reinterpret_cast<volatile const double*>(&sc->partial[i]);
    const double sum = block_sum_fixed(t, s_warp);
    if (threadIdx.x == 0) {
        const double norm = __dsqrt_rn(sum);
        float gs = grad_scale;
        if (clip) {
            const double coef = (double)max_norm / (norm + 1e-6);
            if (coef < 1.0) gs = (float)((double)grad_scale * coef);
        }
        sc->norm = norm;
        sc->gscale_eff = gs;
        if (norm_out) *norm_out = norm;
        sc->counter = 0u;
    }
}

}  // namespace dbuf_k

// Copy-in gather of row-wise FSDP (the baseline the zero-copy bucket
// removes; page section "Importance of zero-copy communication"): each CTA
// moves up to 16384 bf16 gradients of one tensor into its planned place in
// the bucket, scaled by 1/m on the way.  Whole 16-byte granules of the source
// arrive by one bulk copy (TMA, cp.async.bulk) into shared memory; a source
// that is not 16-byte aligned, and the tail, go element by element.
#pragma once

#include <cuda_bf16.h>

#include "tables.h"
#include "tma.cuh"

namespace dbuf_k {

constexpr int kPackThreads = 256;
constexpr int kMaxPackPtrs = 1024;  // tensor pointers passed by value per launch

struct PackPtrs {
    const uint16_t* p[kMaxPackPtrs];
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint16_t scaled_bf16(uint32_t h, float scale) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(bf16_bits_to_f32(h), scale)));
}

__device__ __forceinline__ uint16_t accumulated_bf16(uint32_t d, uint32_t h, float scale) {
    const float t = __fmul_rn(bf16_bits_to_f32(h), scale);
    return __bfloat16_as_ushort(__float2bfloat16_rn(__fadd_rn(bf16_bits_to_f32(d), t)));
}

// ACCUM = false: grad[dst] = bf16(float(src) * scale)           (copy-in)
// ACCUM = true:  grad[dst] = bf16(float(grad[dst]) + float(src) * scale)
//                (gradient accumulation, the DBuffer group add)
template <bool ACCUM>
__global__ void __launch_bounds__(kPackThreads) pack_kernel(PackPtrs ptrs, const PackChunk* __restrict__ chunks,
                                                            int64_t first_chunk, int32_t tensor_base,
                                                            uint16_t* grad, int64_t bucket, float scale,
                                                            int32_t* status) {
    extern __shared__ __align__(128) uint4 sbuf[];
    __shared__ __align__(8) uint64_t bar;
    const PackChunk ch = chunks[first_chunk + blockIdx.x];
    const int32_t ti = ch.tensor - tensor_base;
    if (ti < 0 || ti >= kMaxPackPtrs || ch.count < 0 || ch.count > kPackChunk || ch.dst_off < 0 ||
        ch.dst_off + ch.count > bucket) {
        if (threadIdx.x == 0) set_status(status, 2);
        return;
    }
    const uint16_t* src = ptrs.p[ti] + ch.src_off;
    uint16_t* dst = grad + ch.dst_off;
    const bool aligned = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    const int32_t nbulk = aligned ? (ch.count & ~7) : 0;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar, (uint32_t)nbulk * 2u);
        if (nbulk > 0) bulk_g2s(sbuf, src, (uint32_t)nbulk * 2u, &bar);
    }
    // Element-wise tail while the bulk copy is in flight.
    for (int32_t i = nbulk + threadIdx.x; i < ch.count; i += kPackThreads)
        dst[i] = ACCUM ? accumulated_bf16(dst[i], src[i], scale) : scaled_bf16(src[i], scale);
    if (!mbar_wait_bounded(&bar, 0)) {
        if (threadIdx.x == 0) set_status(status, 1);
        mbar_wait_bounded(&bar, 0);  // let the copy land before the CTA goes away
        return;
    }
    for (int32_t v = threadIdx.x; v < nbulk / 8; v += kPackThreads) {
        const uint4 w = sbuf[v];
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t out[4];
        if (ACCUM) {
            const uint4 dv = *(reinterpret_cast<const uint4*>(dst) + v);
            const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                out[q] = (uint32_t)accumulated_bf16(dw[q] & 0xffffu, in[q] & 0xffffu, scale) |
                         ((uint32_t)accumulated_bf16(dw[q] >> 16, in[q] >> 16, scale) << 16);
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                out[q] = (uint32_t)scaled_bf16(in[q] & 0xffffu, scale) |
                         ((uint32_t)scaled_bf16(in[q] >> 16, scale) << 16);
        }
        __stcs(reinterpret_cast<uint4*>(dst) + v, make_uint4(out[0], out[1], out[2], out[3]));
    }
}

}  // namespace dbuf_k

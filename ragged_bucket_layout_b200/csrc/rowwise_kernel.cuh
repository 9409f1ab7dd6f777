// Interleaved copy-in / copy-out of the row-wise sharded baseline (FSDP2 /
// Megatron-FSDP; veScale-FSDP pages, section on the importance of zero-copy
// communication): the per-parameter copies between each tensor and the
// rank-major communication buffer that the RaggedShard bucket does without.
// One CTA moves one table entry: up to 16384 contiguous elements between a
// tensor and the flat buffer.  When source and destination share their
// position within 16 bytes the body moves in 16-byte vectors (a short
// element-wise head and tail around it); when they share it within 4 bytes,
// in 4-byte words; otherwise element by element.
#pragma once

#include <cuda_bf16.h>

#include "pack_kernel.cuh"
#include "tables.h"
#include "tma.cuh"

namespace dbuf_k {

constexpr int kRowThreads = 256;

template <bool SCALE>
__device__ __forceinline__ uint32_t conv2(uint32_t w, float scale) {
    if (!SCALE) return w;
    return (uint32_t)scaled_bf16(w & 0xffffu, scale) | ((uint32_t)scaled_bf16(w >> 16, scale) << 16);
}

template <bool SCALE>
__device__ __forceinline__ uint16_t conv1(uint16_t h, float scale) {
    return SCALE ? scaled_bf16(h, scale) : h;
}

template <bool SCALE>
__device__ void copy_run(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int32_t n, float scale) {
    const int tid = threadIdx.x;
    const uint32_t as = (uint32_t)reinterpret_cast<uintptr_t>(src) & 15u;
    const uint32_t ad = (uint32_t)reinterpret_cast<uintptr_t>(dst) & 15u;
    if (as == ad) {
        const int32_t head = min(n, (int32_t)(((16u - ad) & 15u) >> 1));
        const int32_t nv = (n - head) >> 3;
        for (int32_t i = tid; i < head; i += kRowThreads) dst[i] = conv1<SCALE>(src[i], scale);
        const uint4* s4 = reinterpret_cast<const uint4*>(src + head);
        uint4* d4 = reinterpret_cast<uint4*>(dst + head);
#pragma unroll 4
        for (int32_t v = tid; v < nv; v += kRowThreads) {
            const uint4 w = __ldcs(s4 + v);
            __stcs(d4 + v, make_uint4(conv2<SCALE>(w.x, scale), conv2<SCALE>(w.y, scale), conv2<SCALE>(w.z, scale),
                                      conv2<SCALE>(w.w, scale)));
        }
        for (int32_t i = head + 8 * nv + tid; i < n; i += kRowThreads) dst[i] = conv1<SCALE>(src[i], scale);
    } else if (((as ^ ad) & 3u) == 0) {
        const int32_t head = min(n, (int32_t)((ad & 3u) >> 1));
        const int32_t nw = (n - head) >> 1;
        for (int32_t i = tid; i < head; i += kRowThreads) dst[i] = conv1<SCALE>(src[i], scale);
        const uint32_t* s2 = reinterpret_cast<const uint32_t*>(src + head);
        uint32_t* d2 = reinterpret_cast<uint32_t*>(dst + head);
#pragma unroll 4
        for (int32_t v = tid; v < nw; v += kRowThreads) __stcs(d2 + v, conv2<SCALE>(__ldcs(s2 + v), scale));
        for (int32_t i = head + 2 * nw + tid; i < n; i += kRowThreads) dst[i] = conv1<SCALE>(src[i], scale);
    } else {
#pragma unroll 4
        for (int32_t i = tid; i < n; i += kRowThreads) dst[i] = conv1<SCALE>(src[i], scale);
    }
}

__device__ void zero_run(uint16_t* dst, int32_t n) {
    const int tid = threadIdx.x;
    const uint32_t ad = (uint32_t)reinterpret_cast<uintptr_t>(dst) & 15u;
    const int32_t head = min(n, (int32_t)(((16u - ad) & 15u) >> 1));
    const int32_t nv = (n - head) >> 3;
    for (int32_t i = tid; i < head; i += kRowThreads) dst[i] = 0;
    uint4* d4 = reinterpret_cast<uint4*>(dst + head);
    for (int32_t v = tid; v < nv; v += kRowThreads) __stcs(d4 + v, make_uint4(0, 0, 0, 0));
    for (int32_t i = head + 8 * nv + tid; i < n; i += kRowThreads) dst[i] = 0;
}

// TO_FLAT = true:  copy-in, flat[dst_off + j] = bf16(float(tensor[src_off + j]) * scale);
//                  entries with tensor < 0 zero flat[dst_off, dst_off + count).
// TO_FLAT = false: copy-out, tensor[src_off + j] = flat[dst_off + j].
// (PackChunk fields: src_off = element offset in the tensor, dst_off = in the flat buffer.)
template <bool TO_FLAT>
__global__ void __launch_bounds__(kRowThreads) rowwise_kernel(PackPtrs ptrs, const PackChunk* __restrict__ chunks,
                                                              int64_t first_chunk, int32_t tensor_base,
                                                              uint16_t* flat, int64_t flat_elems, float scale,
                                                              int32_t* status) {
    const PackChunk ch = chunks[first_chunk + blockIdx.x];
    const bool zero = TO_FLAT && ch.tensor < 0;
    const int32_t ti = ch.tensor - tensor_base;
    if ((!zero && (ti < 0 || ti >= kMaxPackPtrs)) || ch.count < 0 || ch.count > kPackChunk || ch.dst_off < 0 ||
        ch.dst_off + ch.count > flat_elems || ch.src_off < 0) {
        if (threadIdx.x == 0) set_status(status, 2);
        return;
    }
    uint16_t* f = flat + ch.dst_off;
    if (zero) {
        zero_run(f, ch.count);
        return;
    }
    uint16_t* t = const_cast<uint16_t*>(ptrs.p[ti]) + ch.src_off;
    if (TO_FLAT)
        copy_run<true>(t, f, ch.count, scale);
    else
        copy_run<false>(f, t, ch.count, 1.f);
}

}  // namespace dbuf_k

// Row-wise sharded baseline layout (FSDP2 / Megatron-FSDP) and its
// interleaved copy-in / copy-out: the C-ABI's dbuf_rowwise_* functions.
// The layout is what the veScale-FSDP pages compare RaggedShard against
// (comparison of sharding formats; section on the importance of zero-copy
// communication); it exists here to measure the copies RaggedShard saves.
#include <cuda_runtime.h>

#include <algorithm>
#include <new>
#include <string>
#include <vector>

#include "internal.h"
#include "rowwise_kernel.cuh"
#include "tables.h"

using dbuf_detail::fail;
using namespace dbuf_k;

struct dbuf_rowwise_s {
    int32_t n = 0, m = 1;
    int device = 0;
    int64_t chunk = 0;
    std::vector<int64_t> rows, cols, q, off;
    std::vector<int64_t> first;  // first copy entry of each tensor; first[n] = copy entries
    int64_t n_zero = 0;          // zero entries, after the copy entries
    PackChunk* table = nullptr;  // device
    int32_t* status = nullptr;   // device, one word
};

// q_i = ceil(rows_i / m) rows per shard; shards of tensor i start at
// offsets_i within each rank's chunk.
static dbuf_status layout_of(const dbuf_tensor_desc* tensors, int32_t n, int32_t m, dbuf_rowwise_s& rw,
                             const char* who) {
    if (!tensors || n < 1 || m < 1) return fail(DBUF_EINVAL, std::string(who) + ": need n >= 1 tensors and m >= 1");
    rw.n = n;
    rw.m = m;
    int64_t chunk = 0;
    for (int32_t i = 0; i < n; ++i) {
        const dbuf_tensor_desc& d = tensors[i];
        if (d.rows < 1 || d.cols < 1 || d.k < 1 || d.k > d.rows || d.rows > (int64_t(1) << 40) ||
            d.cols > (int64_t(1) << 40) || d.rows * d.cols > (int64_t(1) << 40))
            return fail(DBUF_EINVAL, std::string(who) + ": invalid descriptor " + std::to_string(i));
        const int64_t q = (d.rows + m - 1) / m;
        rw.rows.push_back(d.rows);
        rw.cols.push_back(d.cols);
        rw.q.push_back(q);
        rw.off.push_back(chunk);
        chunk += q * d.cols;
    }
    rw.chunk = chunk;
    if (chunk > (int64_t(1) << 46) / m) return fail(DBUF_EINVAL, std::string(who) + ": gathered buffer too large");
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_rowwise_layout(const dbuf_tensor_desc* tensors, int32_t n, int32_t m,
                                           int64_t* chunk_elems, int64_t* shard_rows, int64_t* offsets) {
    dbuf_rowwise_s rw;
    const dbuf_status s = layout_of(tensors, n, m, rw, "dbuf_rowwise_layout");
    if (s != DBUF_OK) return s;
    if (chunk_elems) *chunk_elems = rw.chunk;
    for (int32_t i = 0; i < n; ++i) {
        if (shard_rows) shard_rows[i] = rw.q[i];
        if (offsets) offsets[i] = rw.off[i];
    }
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_rowwise_create(const dbuf_tensor_desc* tensors, int32_t n, int32_t m, void* stream,
                                           dbuf_rowwise_t** out) {
    if (!out) return fail(DBUF_EINVAL, "dbuf_rowwise_create: out is NULL");
    *out = nullptr;
    dbuf_rowwise_s* rw = new (std::nothrow) dbuf_rowwise_s;
    if (!rw) return fail(DBUF_ENOMEM, "dbuf_rowwise_create: out of host memory");
    {
        const dbuf_status s = layout_of(tensors, n, m, *rw, "dbuf_rowwise_create");
        if (s != DBUF_OK) {
            delete rw;
            return s;
        }
    }
    const int64_t chunk = rw->chunk;
    std::vector<PackChunk> copies, zeros;
    rw->first.assign(n + 1, 0);
    for (int32_t i = 0; i < n; ++i) {
        rw->first[i] = (int64_t)copies.size();
        const int64_t c = rw->cols[i], q = rw->q[i];
        for (int32_t r = 0; r < m; ++r) {
            const int64_t r0 = r * q, r1 = std::max(r0, std::min(rw->rows[i], r0 + q));
            const int64_t len = (r1 - r0) * c, base = r * chunk + rw->off[i];
            for (int64_t e = 0; e < len; e += kPackChunk)
                copies.push_back(PackChunk{r0 * c + e, base + e, i, (int32_t)std::min(kPackChunk, len - e)});
            for (int64_t e = len; e < q * c; e += kPackChunk)
                zeros.push_back(PackChunk{0, base + e, -1, (int32_t)std::min(kPackChunk, q * c - e)});
        }
    }
    rw->first[n] = (int64_t)copies.size();
    rw->n_zero = (int64_t)zeros.size();
    copies.insert(copies.end(), zeros.begin(), zeros.end());
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaGetDevice(&rw->device);
    if (e == cudaSuccess) e = cudaMalloc(&rw->status, 256 + std::max<size_t>(1, copies.size()) * sizeof(PackChunk));
    if (e == cudaSuccess) {
        rw->table = reinterpret_cast<PackChunk*>(reinterpret_cast<char*>(rw->status) + 256);
        e = cudaMemsetAsync(rw->status, 0, 256, st);
    }
    if (e == cudaSuccess && !copies.empty())
        e = cudaMemcpyAsync(rw->table, copies.data(), copies.size() * sizeof(PackChunk), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);  // `copies` is released on return
    if (e != cudaSuccess) {
        if (rw->status) cudaFree(rw->status);
        delete rw;
        return fail(DBUF_ECUDA, std::string("dbuf_rowwise_create: ") + cudaGetErrorString(e));
    }
    *out = rw;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_rowwise_info(const dbuf_rowwise_t* rw, int64_t* chunk_elems, int64_t* shard_rows,
                                         int64_t* offsets) {
    if (!rw) return fail(DBUF_EINVAL, "dbuf_rowwise_info: rw is NULL");
    if (chunk_elems) *chunk_elems = rw->chunk;
    for (int32_t i = 0; i < rw->n; ++i) {
        if (shard_rows) shard_rows[i] = rw->q[i];
        if (offsets) offsets[i] = rw->off[i];
    }
    return DBUF_OK;
}

template <bool TO_FLAT>
static dbuf_status rowwise_launch(dbuf_rowwise_t* rw, const void* const* ptrs, void* flat, float scale,
                                  void* stream, const char* who) {
    if (!rw) return fail(DBUF_EINVAL, std::string(who) + ": rw is NULL");
    if (!ptrs || !flat) return fail(DBUF_EINVAL, std::string(who) + ": NULL buffer");
    if (reinterpret_cast<uintptr_t>(flat) & 1u) return fail(DBUF_EINVAL, std::string(who) + ": flat buffer not 2-byte aligned");
    for (int32_t i = 0; i < rw->n; ++i)
        if (!ptrs[i] || (reinterpret_cast<uintptr_t>(ptrs[i]) & 1u))
            return fail(DBUF_EINVAL, std::string(who) + ": tensor pointer " + std::to_string(i) + " NULL or not 2-byte aligned");
    int dev = -1;
    CUDA_TRY(cudaGetDevice(&dev), who);
    if (dev != rw->device) return fail(DBUF_EINVAL, std::string(who) + ": wrong current device");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint16_t* f = static_cast<uint16_t*>(flat);
    const int64_t flat_elems = rw->chunk * rw->m;
    for (int32_t t0 = 0; t0 < rw->n; t0 += kMaxPackPtrs) {
        const int32_t t1 = std::min<int32_t>(rw->n, t0 + kMaxPackPtrs);
        const int64_t c0 = rw->first[t0], c1 = rw->first[t1];
        if (c1 == c0) continue;
        PackPtrs pp{};
        for (int32_t i = t0; i < t1; ++i) pp.p[i - t0] = static_cast<const uint16_t*>(ptrs[i]);
        for (int64_t c = c0; c < c1; c += 0x7fffffff) {
            const unsigned grid = (unsigned)std::min<int64_t>(c1 - c, 0x7fffffff);
            rowwise_kernel<TO_FLAT><<<grid, kRowThreads, 0, st>>>(pp, rw->table, c, t0, f, flat_elems, scale, rw->status);
            CUDA_TRY(cudaGetLastError(), std::string(who) + ": launch");
        }
    }
    if (TO_FLAT && rw->n_zero > 0) {
        PackPtrs none{};
        const int64_t c0 = rw->first[rw->n];
        rowwise_kernel<true><<<(unsigned)rw->n_zero, kRowThreads, 0, st>>>(none, rw->table, c0, 0, f, flat_elems, 0.f,
                                                                           rw->status);
        CUDA_TRY(cudaGetLastError(), std::string(who) + ": zero launch");
    }
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_rowwise_copy_out(dbuf_rowwise_t* rw, const void* gathered_bf16, void* const* params_bf16,
                                             void* stream) {
    return rowwise_launch<false>(rw, const_cast<const void* const*>(params_bf16), const_cast<void*>(gathered_bf16),
                                 1.f, stream, "dbuf_rowwise_copy_out");
}

extern "C" dbuf_status dbuf_rowwise_copy_in(dbuf_rowwise_t* rw, const void* const* grads_bf16, float scale,
                                            void* rs_input_bf16, void* stream) {
    return rowwise_launch<true>(rw, grads_bf16, rs_input_bf16, scale, stream, "dbuf_rowwise_copy_in");
}

extern "C" dbuf_status dbuf_rowwise_status(dbuf_rowwise_t* rw, int32_t* code, void* stream) {
    if (!rw || !code) return fail(DBUF_EINVAL, "dbuf_rowwise_status: NULL argument");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    CUDA_TRY(cudaMemcpyAsync(code, rw->status, sizeof(int32_t), cudaMemcpyDeviceToHost, st), "dbuf_rowwise_status");
    CUDA_TRY(cudaStreamSynchronize(st), "dbuf_rowwise_status");
    return DBUF_OK;
}

extern "C" void dbuf_rowwise_destroy(dbuf_rowwise_t* rw) {
    if (!rw) return;
    if (rw->status) cudaFree(rw->status);
    delete rw;
}

// Device runtime of the ragged-bucket optimizer step (sm_100a).
//
// DBuffer (veScale-FSDP paper Sec. 5, page section "3. DBuffer"): one batch
// allocation holds every bucket array of a plan; tensors are zero-copy views;
// group operations run as one launch over the whole bucket.  The fused step
// is the block-wise 8-bit Adam of the paper's 8-bit Adam case study
// (Sec. 6.3): each quantisation block (k whole rows) is updated and
// requantised on its own, which the RaggedShard layout makes possible
// because no block crosses a slice boundary.
//
// Work decomposition (host-built table, uploaded once by dbuf_create):
//   WHOLE  up to 4096 elements holding up to 256 whole blocks of one tensor;
//          one CTA keeps the new m and sqrt(v) in registers, reduces each
//          block's absmax in shared memory, then writes the codes.
//   LARGE  one block longer than a tile; one CTA streams it twice: pass 1
//          updates weights and finds the absmax, pass 2 re-reads grad and
//          codes (an L2 hit while the block is recent), recomputes m and
//          sqrt(v) bit-identically and writes the codes.
//   ZERO   a padding range; the bf16 parameter copy is set to zero.
// Every thread owns 16 consecutive elements (16-element aligned in the
// bucket), so grad, master, codes and the bf16 copy move as 128-bit accesses.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "internal.h"

// ------------------------------------------------------------------ errors

namespace dbuf_detail {
static thread_local std::string g_err;
void set_error(const std::string& msg) { g_err = msg; }
dbuf_status fail(dbuf_status st, const std::string& msg) {
    g_err = msg;
    return st;
}
}  // namespace dbuf_detail

using dbuf_detail::fail;

extern "C" const char* dbuf_last_error(void) { return dbuf_detail::g_err.c_str(); }

#define CUDA_TRY(call, what)                                                                  \
    do {                                                                                      \
        cudaError_t e_ = (call);                                                              \
        if (e_ != cudaSuccess)                                                                \
            return fail(DBUF_ECUDA, std::string(what) + ": " + cudaGetErrorString(e_));       \
    } while (0)

// ------------------------------------------------------------ work tables

namespace {

constexpr int kThreads = 256;          // threads per CTA of the step kernel
constexpr int kVec = 16;               // elements per thread-vector
constexpr int kTile = kThreads * kVec; // 4096 elements per tile
constexpr int kMaxBlk = 256;           // blocks per WHOLE tile
constexpr int64_t kZeroChunk = 65536;  // elements per ZERO tile
constexpr int64_t kPackChunk = 16384;  // elements per copy-in CTA (32 KB)
constexpr int kPackThreads = 256;
constexpr int kMaxPackPtrs = 1024;     // tensor pointers passed by value per launch

enum : int32_t { TILE_WHOLE = 0, TILE_LARGE = 1, TILE_ZERO = 2 };

struct Tile {
    int64_t e0;    // first bucket element of the tile
    int64_t blk0;  // index of its first block (scale index)
    int64_t n;     // elements in the tile
    int32_t b;     // block size (WHOLE), 0 otherwise
    int32_t kind;
    int32_t nblk;  // blocks in the tile (WHOLE)
    int32_t pad_;
};
static_assert(sizeof(Tile) == 40, "tile layout");

struct PackChunk {
    int64_t src_off;  // element offset in the source tensor
    int64_t dst_off;  // element offset in the bucket
    int32_t tensor;   // caller's tensor index
    int32_t count;    // elements
};

struct PackPtrs {
    const uint16_t* p[kMaxPackPtrs];
};

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

void add_zero_tiles(std::vector<Tile>& out, int64_t a, int64_t b) {
    for (int64_t e = a; e < b; e += kZeroChunk)
        out.push_back(Tile{e, 0, std::min(kZeroChunk, b - e), 0, TILE_ZERO, 0, 0});
}

void build_tiles(const dbuf_plan_s& p, std::vector<Tile>& tiles) {
    std::vector<Tile> large, whole, zero;
    int64_t blk = 0, prev_end = 0;
    for (int32_t id : p.by_offset) {
        const int64_t o = p.offset[id], n = p.rows[id] * p.cols[id], b = p.k[id] * p.cols[id];
        const int64_t nb = cdiv(p.rows[id], p.k[id]);
        if (o > prev_end) add_zero_tiles(zero, prev_end, o);
        int64_t j = 0;
        while (j < nb) {
            const int64_t e0 = o + j * b;
            if (b <= kTile) {
                const int64_t cap = kTile - (e0 & (kVec - 1));
                const int64_t q = std::min<int64_t>({kMaxBlk, cap / b, nb - j});
                if (q >= 1) {
                    whole.push_back(Tile{e0, blk + j, std::min(q * b, n - j * b), (int32_t)b, TILE_WHOLE,
                                         (int32_t)q, 0});
                    j += q;
                    continue;
                }
            }
            large.push_back(Tile{e0, blk + j, std::min(b, n - j * b), 0, TILE_LARGE, 1, 0});
            j += 1;
        }
        blk += nb;
        prev_end = o + n;
    }
    if (prev_end < p.bucket) add_zero_tiles(zero, prev_end, p.bucket);
    // Longest work first so the tail of the grid is short tiles.
    std::stable_sort(large.begin(), large.end(), [](const Tile& x, const Tile& y) { return x.n > y.n; });
    tiles.clear();
    tiles.reserve(large.size() + whole.size() + zero.size());
    tiles.insert(tiles.end(), large.begin(), large.end());
    tiles.insert(tiles.end(), whole.begin(), whole.end());
    tiles.insert(tiles.end(), zero.begin(), zero.end());
}

void build_pack_chunks(const dbuf_plan_s& p, std::vector<PackChunk>& chunks, std::vector<int64_t>& first) {
    chunks.clear();
    first.assign(p.n + 1, 0);
    for (int32_t i = 0; i < p.n; ++i) {
        first[i] = (int64_t)chunks.size();
        const int64_t n = p.rows[i] * p.cols[i];
        for (int64_t e = 0; e < n; e += kPackChunk)
            chunks.push_back(PackChunk{e, p.offset[i] + e, i, (int32_t)std::min(kPackChunk, n - e)});
    }
    first[p.n] = (int64_t)chunks.size();
}

struct Layout {
    size_t master, param, grad, mq, vq, scales, tiles, chunks, status, total;
};

Layout layout_of(const dbuf_plan_s& p, size_t n_tiles, size_t n_chunks) {
    Layout L{};
    const size_t S = (size_t)p.bucket;
    size_t at = 0;
    L.master = at; at = align256(at + S * 4);
    L.param = at;  at = align256(at + S * 2);
    L.grad = at;   at = align256(at + S * 2);
    L.mq = at;     at = align256(at + S);
    L.vq = at;     at = align256(at + S);
    L.scales = at; at = align256(at + ((size_t)p.n_blocks + 2) * 8);
    L.tiles = at;  at = align256(at + n_tiles * sizeof(Tile));
    L.chunks = at; at = align256(at + n_chunks * sizeof(PackChunk));
    L.status = at; at = align256(at + 16);
    L.total = at;
    return L;
}

}  // namespace

struct dbuf_s {
    dbuf_plan_s plan;
    int device = -1;
    char* base = nullptr;
    size_t bytes = 0;
    bool owns = false;
    Layout lay{};
    float* master = nullptr;
    uint16_t* param = nullptr;
    uint16_t* grad = nullptr;
    int8_t* mq = nullptr;
    uint8_t* vq = nullptr;
    float2* scales = nullptr;
    Tile* tiles = nullptr;
    PackChunk* chunks = nullptr;
    int32_t* status = nullptr;
    std::vector<Tile> h_tiles;
    std::vector<PackChunk> h_chunks;
    std::vector<int64_t> h_chunk_first;
};

// ----------------------------------------------------------- device code

namespace {

struct StepC {
    float b1, omb1, b2, omb2, bc2s, eps, step, decay, gscale;
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ void set_status(int32_t* status, int32_t code) { atomicCAS(status, 0, code); }

// New m and sqrt(v) of one element, every operation rounded on its own.
__device__ __forceinline__ void new_m_r(float graw, float qm, float qv, float dqm, float dqv,
                                        const StepC& c, float& m, float& r) {
    const float g = __fmul_rn(graw, c.gscale);
    const float mo = __fmul_rn(qm, dqm);
    const float so = __fmul_rn(qv, dqv);
    const float vo = __fmul_rn(so, so);
    m = __fadd_rn(__fmul_rn(c.b1, mo), __fmul_rn(c.omb1, g));
    const float gg = __fmul_rn(g, g);
    const float v = __fadd_rn(__fmul_rn(c.b2, vo), __fmul_rn(c.omb2, gg));
    r = __fsqrt_rn(v);
}

__device__ __forceinline__ float new_p(float p, float m, float r, const StepC& c) {
    const float d = __fadd_rn(__fdiv_rn(r, c.bc2s), c.eps);
    const float u = __fdiv_rn(m, d);
    return __fsub_rn(__fmul_rn(p, c.decay), __fmul_rn(c.step, u));
}

__device__ __forceinline__ uint32_t code_m(float m, float q) {
    float a = rintf(__fmul_rn(m, q));
    a = fminf(127.f, fmaxf(-127.f, a));
    return (uint32_t)((int32_t)a) & 0xffu;
}

__device__ __forceinline__ uint32_t code_v(float r, float q) {
    float b = rintf(__fmul_rn(r, q));
    b = fminf(255.f, fmaxf(0.f, b));
    return (uint32_t)b;
}

// Registers of one thread-vector: 16 consecutive bucket elements.
struct Vec16 {
    uint32_t g[8];   // bf16 pairs
    float p[16];
    uint32_t mq[4];  // 16 int8 codes
    uint32_t vq[4];  // 16 uint8 codes
};

__device__ __forceinline__ uint32_t byte_of(const uint32_t* w, int i) { return (w[i >> 2] >> (8 * (i & 3))) & 0xffu; }
__device__ __forceinline__ float gval(const uint32_t* g, int i) { return bf16_bits_to_f32((g[i >> 1] >> (16 * (i & 1))) & 0xffffu); }

// Load elements [vb, vb+16) clipped to [lo, hi); out-of-range lanes read 0.
__device__ __forceinline__ void load_vec(Vec16& x, int64_t vb, int64_t lo, int64_t hi, bool full, bool want_p,
                                         const float* master, const uint16_t* grad, const int8_t* mq,
                                         const uint8_t* vq) {
    if (full) {
        const uint4 g0 = __ldg(reinterpret_cast<const uint4*>(grad + vb));
        const uint4 g1 = __ldg(reinterpret_cast<const uint4*>(grad + vb) + 1);
        x.g[0] = g0.x; x.g[1] = g0.y; x.g[2] = g0.z; x.g[3] = g0.w;
        x.g[4] = g1.x; x.g[5] = g1.y; x.g[6] = g1.z; x.g[7] = g1.w;
        const uint4 a = *reinterpret_cast<const uint4*>(mq + vb);
        const uint4 b = *reinterpret_cast<const uint4*>(vq + vb);
        x.mq[0] = a.x; x.mq[1] = a.y; x.mq[2] = a.z; x.mq[3] = a.w;
        x.vq[0] = b.x; x.vq[1] = b.y; x.vq[2] = b.z; x.vq[3] = b.w;
        if (want_p) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 f = __ldcs(reinterpret_cast<const float4*>(master + vb) + q);
                x.p[4 * q] = f.x; x.p[4 * q + 1] = f.y; x.p[4 * q + 2] = f.z; x.p[4 * q + 3] = f.w;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x.g[i] = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) x.mq[i] = x.vq[i] = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int64_t e = vb + i;
            const bool in = (e >= lo && e < hi);
            x.p[i] = (in && want_p) ? master[e] : 0.f;
            if (in) {
                x.g[i >> 1] |= (uint32_t)grad[e] << (16 * (i & 1));
                x.mq[i >> 2] |= ((uint32_t)(uint8_t)mq[e]) << (8 * (i & 3));
                x.vq[i >> 2] |= ((uint32_t)vq[e]) << (8 * (i & 3));
            }
        }
    }
}

__device__ __forceinline__ void store_p_bf16(const float* p, int64_t vb, int64_t lo, int64_t hi, bool full,
                                             float* master, uint16_t* param) {
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(p[2 * i]));
        const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(p[2 * i + 1]));
        h[i] = a | (b << 16);
    }
    if (full) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            __stcs(reinterpret_cast<float4*>(master + vb) + q,
                   make_float4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]));
        __stcs(reinterpret_cast<uint4*>(param + vb), make_uint4(h[0], h[1], h[2], h[3]));
        __stcs(reinterpret_cast<uint4*>(param + vb) + 1, make_uint4(h[4], h[5], h[6], h[7]));
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int64_t e = vb + i;
            if (e >= lo && e < hi) {
                master[e] = p[i];
                param[e] = (uint16_t)((h[i >> 1] >> (16 * (i & 1))) & 0xffffu);
            }
        }
    }
}

__device__ __forceinline__ void store_codes(const uint32_t* cm, const uint32_t* cv, int64_t vb, int64_t lo,
                                            int64_t hi, bool full, int8_t* mq, uint8_t* vq) {
    if (full) {
        __stcs(reinterpret_cast<uint4*>(mq + vb), make_uint4(cm[0], cm[1], cm[2], cm[3]));
        __stcs(reinterpret_cast<uint4*>(vq + vb), make_uint4(cv[0], cv[1], cv[2], cv[3]));
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int64_t e = vb + i;
            if (e >= lo && e < hi) {
                mq[e] = (int8_t)byte_of(cm, i);
                vq[e] = (uint8_t)byte_of(cv, i);
            }
        }
    }
}

// Max over the lanes of a warp that share `key`, where lanes with equal keys
// are contiguous; the first lane of each run gets the run's maximum.
__device__ __forceinline__ void segmented_max(int key, uint32_t& a, uint32_t& b, bool& head) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int ok = __shfl_down_sync(0xffffffffu, key, d);
        const uint32_t oa = __shfl_down_sync(0xffffffffu, a, d);
        const uint32_t ob = __shfl_down_sync(0xffffffffu, b, d);
        if (lane + d < 32 && ok == key) {
            a = max(a, oa);
            b = max(b, ob);
        }
    }
    const int prev = __shfl_up_sync(0xffffffffu, key, 1);
    head = (lane == 0) || (prev != key);
}

__device__ void whole_tile(const Tile& t, float* master, uint16_t* param, const uint16_t* grad, int8_t* mq,
                           uint8_t* vq, float2* scales, const StepC& c) {
    __shared__ float s_dqm[kMaxBlk], s_dqv[kMaxBlk], s_qm[kMaxBlk], s_qv[kMaxBlk];
    __shared__ uint32_t s_am[kMaxBlk], s_ar[kMaxBlk];
    const int tid = threadIdx.x;
    if (tid < t.nblk) {
        const float2 sc = scales[t.blk0 + tid];
        s_dqm[tid] = __fdiv_rn(sc.x, 127.f);
        s_dqv[tid] = __fdiv_rn(sc.y, 255.f);
        s_am[tid] = 0u;
        s_ar[tid] = 0u;
    }
    __syncthreads();

    const int64_t lo = t.e0, hi = t.e0 + t.n;
    const int64_t vb = (t.e0 & ~int64_t(kVec - 1)) + (int64_t)kVec * tid;
    const int64_t elo = max(vb, lo), ehi = min(vb + kVec, hi);
    const bool any = elo < ehi;
    const bool full = (elo == vb) && (ehi == vb + kVec);
    const int32_t b = t.b;

    Vec16 x;
    float m[16], r[16];
    int blk_first = -1, blk_last = -1;
    if (any) {
        load_vec(x, vb, lo, hi, full, true, master, grad, mq, vq);
        blk_first = (int)((elo - lo) / b);
        blk_last = (int)((ehi - 1 - lo) / b);
        const bool one = (blk_first == blk_last);
        const float dqm1 = s_dqm[blk_first], dqv1 = s_dqv[blk_first];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float dqm = dqm1, dqv = dqv1;
            if (!one) {
                const int64_t e = vb + i;
                const int lb = (e >= lo && e < hi) ? (int)((e - lo) / b) : blk_first;
                dqm = s_dqm[lb];
                dqv = s_dqv[lb];
            }
            new_m_r(gval(x.g, i), (float)(int8_t)byte_of(x.mq, i), (float)byte_of(x.vq, i), dqm, dqv, c, m[i], r[i]);
            x.p[i] = new_p(x.p[i], m[i], r[i], c);
        }
        store_p_bf16(x.p, vb, lo, hi, full, master, param);
    }

    // Per-block absmax of |m| and r (non-negative floats compare as integers).
    const bool one = any && (blk_first == blk_last);
    uint32_t am = 0u, ar = 0u;
    if (one) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int64_t e = vb + i;
            if (full || (e >= lo && e < hi)) {
                am = max(am, __float_as_uint(fabsf(m[i])));
                ar = max(ar, __float_as_uint(r[i]));
            }
        }
    } else if (any) {
        for (int i = 0; i < 16; ++i) {
            const int64_t e = vb + i;
            if (e >= lo && e < hi) {
                const int lb = (int)((e - lo) / b);
                atomicMax(&s_am[lb], __float_as_uint(fabsf(m[i])));
                atomicMax(&s_ar[lb], __float_as_uint(r[i]));
            }
        }
    }
    bool head;
    const int key = one ? blk_first : -1;
    segmented_max(key, am, ar, head);
    if (one && head) {
        atomicMax(&s_am[key], am);
        atomicMax(&s_ar[key], ar);
    }
    __syncthreads();
    if (tid < t.nblk) {
        const float AMm = __uint_as_float(s_am[tid]), AMr = __uint_as_float(s_ar[tid]);
        s_qm[tid] = AMm > 0.f ? __fdiv_rn(127.f, AMm) : 0.f;
        s_qv[tid] = AMr > 0.f ? __fdiv_rn(255.f, AMr) : 0.f;
        scales[t.blk0 + tid] = make_float2(AMm, AMr);
    }
    __syncthreads();
    if (any) {
        uint32_t cm[4] = {0, 0, 0, 0}, cv[4] = {0, 0, 0, 0};
        const float qm1 = s_qm[blk_first], qv1 = s_qv[blk_first];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float qm = qm1, qv = qv1;
            if (!one) {
                const int64_t e = vb + i;
                const int lb = (e >= lo && e < hi) ? (int)((e - lo) / b) : blk_first;
                qm = s_qm[lb];
                qv = s_qv[lb];
            }
            cm[i >> 2] |= code_m(m[i], qm) << (8 * (i & 3));
            cv[i >> 2] |= code_v(r[i], qv) << (8 * (i & 3));
        }
        store_codes(cm, cv, vb, lo, hi, full, mq, vq);
    }
}

__device__ void large_block(const Tile& t, float* master, uint16_t* param, const uint16_t* grad, int8_t* mq,
                            uint8_t* vq, float2* scales, const StepC& c) {
    __shared__ uint32_t s_red[2][kThreads / 32];
    __shared__ float s_q[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float2 sc = scales[t.blk0];
    const float dqm = __fdiv_rn(sc.x, 127.f), dqv = __fdiv_rn(sc.y, 255.f);
    const int64_t lo = t.e0, hi = t.e0 + t.n;
    const int64_t a0 = t.e0 & ~int64_t(kVec - 1);

    // Pass 1: full update, weights written, absmax accumulated.
    uint32_t am = 0u, ar = 0u;
    for (int64_t vb = a0 + (int64_t)kVec * tid; vb < hi; vb += kTile) {
        const int64_t elo = max(vb, lo), ehi = min(vb + kVec, hi);
        const bool full = (elo == vb) && (ehi == vb + kVec);
        Vec16 x;
        load_vec(x, vb, lo, hi, full, true, master, grad, mq, vq);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float m, r;
            new_m_r(gval(x.g, i), (float)(int8_t)byte_of(x.mq, i), (float)byte_of(x.vq, i), dqm, dqv, c, m, r);
            x.p[i] = new_p(x.p[i], m, r, c);
            const int64_t e = vb + i;
            if (full || (e >= lo && e < hi)) {
                am = max(am, __float_as_uint(fabsf(m)));
                ar = max(ar, __float_as_uint(r));
            }
        }
        store_p_bf16(x.p, vb, lo, hi, full, master, param);
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        am = max(am, __shfl_xor_sync(0xffffffffu, am, d));
        ar = max(ar, __shfl_xor_sync(0xffffffffu, ar, d));
    }
    if (lane == 0) {
        s_red[0][warp] = am;
        s_red[1][warp] = ar;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t a = 0u, bb = 0u;
        for (int w = 0; w < kThreads / 32; ++w) {
            a = max(a, s_red[0][w]);
            bb = max(bb, s_red[1][w]);
        }
        const float AMm = __uint_as_float(a), AMr = __uint_as_float(bb);
        s_q[0] = AMm > 0.f ? __fdiv_rn(127.f, AMm) : 0.f;
        s_q[1] = AMr > 0.f ? __fdiv_rn(255.f, AMr) : 0.f;
        scales[t.blk0] = make_float2(AMm, AMr);
    }
    __syncthreads();
    const float qm = s_q[0], qv = s_q[1];

    // Pass 2: recompute m and sqrt(v) from the unchanged grad and old codes.
    for (int64_t vb = a0 + (int64_t)kVec * tid; vb < hi; vb += kTile) {
        const int64_t elo = max(vb, lo), ehi = min(vb + kVec, hi);
        const bool full = (elo == vb) && (ehi == vb + kVec);
        Vec16 x;
        load_vec(x, vb, lo, hi, full, false, master, grad, mq, vq);
        uint32_t cm[4] = {0, 0, 0, 0}, cv[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float m, r;
            new_m_r(gval(x.g, i), (float)(int8_t)byte_of(x.mq, i), (float)byte_of(x.vq, i), dqm, dqv, c, m, r);
            cm[i >> 2] |= code_m(m, qm) << (8 * (i & 3));
            cv[i >> 2] |= code_v(r, qv) << (8 * (i & 3));
        }
        store_codes(cm, cv, vb, lo, hi, full, mq, vq);
    }
}

__device__ void zero_tile(const Tile& t, uint16_t* param) {
    const int64_t lo = t.e0, hi = t.e0 + t.n;
    const int64_t a0 = t.e0 & ~int64_t(kVec - 1);
    for (int64_t vb = a0 + (int64_t)kVec * threadIdx.x; vb < hi; vb += kTile) {
        if (vb >= lo && vb + kVec <= hi) {
            uint4* q = reinterpret_cast<uint4*>(param + vb);
            __stcs(q, make_uint4(0, 0, 0, 0));
            __stcs(q + 1, make_uint4(0, 0, 0, 0));
        } else {
            for (int i = 0; i < kVec; ++i)
                if (vb + i >= lo && vb + i < hi) param[vb + i] = 0;
        }
    }
}

__global__ void __launch_bounds__(kThreads) adam8_step_kernel(const Tile* __restrict__ tiles, int64_t n_tiles,
                                                              int64_t bucket, float* master, uint16_t* param,
                                                              const uint16_t* __restrict__ grad, int8_t* mq,
                                                              uint8_t* vq, float2* scales, int64_t n_blocks,
                                                              StepC c, int32_t* status) {
    if ((int64_t)blockIdx.x >= n_tiles) return;
    const Tile t = tiles[blockIdx.x];
    // Bounds of the table entry against the bucket; a bad entry is reported,
    // never accessed.
    if (t.e0 < 0 || t.n < 0 || t.e0 + t.n > bucket ||
        (t.kind != TILE_ZERO && (t.blk0 < 0 || t.blk0 + t.nblk > n_blocks)) ||
        (t.kind == TILE_WHOLE && (t.b <= 0 || t.nblk > kMaxBlk || (t.e0 & (kVec - 1)) + t.n > kTile))) {
        if (threadIdx.x == 0) set_status(status, 2);
        return;
    }
    if (t.kind == TILE_WHOLE)
        whole_tile(t, master, param, grad, mq, vq, scales, c);
    else if (t.kind == TILE_LARGE)
        large_block(t, master, param, grad, mq, vq, scales, c);
    else
        zero_tile(t, param);
}

// ------------------------------------------------------- copy-in (TMA bulk)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for an mbarrier phase, giving up after ~limit_ns; false on time-out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u && global_ns() - t0 > limit_ns) return false;
    }
}

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: far beyond any copy

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
    // Whole 16-byte granules go through one bulk copy into shared memory.
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
    // Scalar tail while the bulk copy is in flight.
    for (int32_t i = nbulk + threadIdx.x; i < ch.count; i += kPackThreads) {
        const float f = __fmul_rn(bf16_bits_to_f32(src[i]), scale);
        dst[i] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
    }
    if (!mbar_wait_bounded(&bar, 0, kWaitNs)) {
        if (threadIdx.x == 0) set_status(status, 1);
        // Let the copy land before the CTA (and its shared memory) goes away.
        mbar_wait_bounded(&bar, 0, kWaitNs);
        return;
    }
    for (int32_t v = threadIdx.x; v < nbulk / 8; v += kPackThreads) {
        const uint4 w = sbuf[v];
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo_f = __fmul_rn(bf16_bits_to_f32(in[q] & 0xffffu), scale);
            const float hi_f = __fmul_rn(bf16_bits_to_f32(in[q] >> 16), scale);
            out[q] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo_f)) |
                     ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi_f)) << 16);
        }
        __stcs(reinterpret_cast<uint4*>(dst) + v, make_uint4(out[0], out[1], out[2], out[3]));
    }
}

StepC make_step_constants(const dbuf_adam_hparams& hp, float grad_scale) {
    const double B1 = hp.beta1, B2 = hp.beta2, lr = hp.lr, wd = hp.weight_decay, t = (double)hp.step;
    const double bc1 = 1.0 - std::pow(B1, t);
    const double bc2 = 1.0 - std::pow(B2, t);
    StepC c;
    c.b1 = (float)B1;
    c.omb1 = (float)(1.0 - B1);
    c.b2 = (float)B2;
    c.omb2 = (float)(1.0 - B2);
    c.bc2s = (float)std::sqrt(bc2);
    c.eps = hp.eps;
    c.step = (float)(lr / bc1);
    c.decay = (float)(1.0 - lr * wd);
    c.gscale = grad_scale;
    return c;
}

dbuf_status check_device(const dbuf_t* db, const char* who) {
    int dev = -1;
    CUDA_TRY(cudaGetDevice(&dev), who);
    if (dev != db->device)
        return fail(DBUF_EINVAL, std::string(who) + ": current device " + std::to_string(dev) +
                                     " is not the dbuf's device " + std::to_string(db->device));
    return DBUF_OK;
}

}  // namespace

// ------------------------------------------------------------------- C-ABI

extern "C" size_t dbuf_required_bytes(const dbuf_plan_t* plan) {
    if (!plan) return 0;
    std::vector<Tile> tiles;
    build_tiles(*plan, tiles);
    std::vector<PackChunk> chunks;
    std::vector<int64_t> first;
    build_pack_chunks(*plan, chunks, first);
    return layout_of(*plan, tiles.size(), chunks.size()).total;
}

extern "C" dbuf_status dbuf_work_table(const dbuf_plan_t* plan, dbuf_work_item* out, int64_t cap, int64_t* n) {
    if (!plan || !n) return fail(DBUF_EINVAL, "dbuf_work_table: NULL argument");
    if (cap > 0 && !out) return fail(DBUF_EINVAL, "dbuf_work_table: out is NULL");
    std::vector<Tile> tiles;
    build_tiles(*plan, tiles);
    *n = (int64_t)tiles.size();
    static_assert(sizeof(dbuf_work_item) == sizeof(Tile), "work item mirrors the device tile");
    const int64_t m = std::min<int64_t>(cap, *n);
    for (int64_t i = 0; i < m; ++i)
        out[i] = dbuf_work_item{tiles[i].e0, tiles[i].blk0, tiles[i].n, tiles[i].b, tiles[i].kind, tiles[i].nblk, 0};
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_create(const dbuf_plan_t* plan, void* device_base, size_t base_bytes, void* stream,
                                   dbuf_t** out) {
    if (!out) return fail(DBUF_EINVAL, "dbuf_create: out is NULL");
    *out = nullptr;
    if (!plan) return fail(DBUF_EINVAL, "dbuf_create: plan is NULL");
    if (plan->align % kVec != 0)
        return fail(DBUF_EINVAL, "dbuf_create: plan alignment must be a multiple of 16 elements");
    dbuf_s* db = new (std::nothrow) dbuf_s;
    if (!db) return fail(DBUF_ENOMEM, "dbuf_create: out of host memory");
    db->plan = *plan;
    build_tiles(db->plan, db->h_tiles);
    build_pack_chunks(db->plan, db->h_chunks, db->h_chunk_first);
    db->lay = layout_of(db->plan, db->h_tiles.size(), db->h_chunks.size());
    db->bytes = db->lay.total;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaGetDevice(&db->device);
    if (e != cudaSuccess) {
        delete db;
        return fail(DBUF_ECUDA, std::string("dbuf_create: cudaGetDevice: ") + cudaGetErrorString(e));
    }
    if (device_base) {
        if ((reinterpret_cast<uintptr_t>(device_base) & 255u) != 0 || base_bytes < db->bytes) {
            const size_t need = db->bytes;
            delete db;
            return fail(DBUF_EINVAL, "dbuf_create: device_base must be 256-byte aligned and at least " +
                                         std::to_string(need) + " bytes");
        }
        db->base = static_cast<char*>(device_base);
        db->owns = false;
    } else {
        void* p = nullptr;
        e = cudaMalloc(&p, db->bytes);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            const size_t need = db->bytes;
            delete db;
            return fail(DBUF_ENOMEM, "dbuf_create: cudaMalloc of " + std::to_string(need) +
                                         " bytes failed: " + cudaGetErrorString(e));
        }
        db->base = static_cast<char*>(p);
        db->owns = true;
    }
    char* b = db->base;
    db->master = reinterpret_cast<float*>(b + db->lay.master);
    db->param = reinterpret_cast<uint16_t*>(b + db->lay.param);
    db->grad = reinterpret_cast<uint16_t*>(b + db->lay.grad);
    db->mq = reinterpret_cast<int8_t*>(b + db->lay.mq);
    db->vq = reinterpret_cast<uint8_t*>(b + db->lay.vq);
    db->scales = reinterpret_cast<float2*>(b + db->lay.scales);
    db->tiles = reinterpret_cast<Tile*>(b + db->lay.tiles);
    db->chunks = reinterpret_cast<PackChunk*>(b + db->lay.chunks);
    db->status = reinterpret_cast<int32_t*>(b + db->lay.status);
    e = cudaMemsetAsync(db->base, 0, db->bytes, st);
    if (e == cudaSuccess && !db->h_tiles.empty())
        e = cudaMemcpyAsync(db->tiles, db->h_tiles.data(), db->h_tiles.size() * sizeof(Tile),
                            cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess && !db->h_chunks.empty())
        e = cudaMemcpyAsync(db->chunks, db->h_chunks.data(), db->h_chunks.size() * sizeof(PackChunk),
                            cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) {
        if (db->owns) cudaFree(db->base);
        delete db;
        return fail(DBUF_ECUDA, std::string("dbuf_create: initialising the bucket: ") + cudaGetErrorString(e));
    }
    *out = db;
    return DBUF_OK;
}

extern "C" void dbuf_destroy(dbuf_t* db) {
    if (!db) return;
    if (db->owns && db->base) cudaFree(db->base);
    delete db;
}

extern "C" dbuf_status dbuf_pack_grads(dbuf_t* db, const void* const* grads_bf16, float scale, void* stream) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_pack_grads: db is NULL");
    if (db->plan.n > 0 && !grads_bf16) return fail(DBUF_EINVAL, "dbuf_pack_grads: grads_bf16 is NULL");
    for (int32_t i = 0; i < db->plan.n; ++i)
        if (!grads_bf16[i] || (reinterpret_cast<uintptr_t>(grads_bf16[i]) & 1u))
            return fail(DBUF_EINVAL, "dbuf_pack_grads: gradient pointer " + std::to_string(i) +
                                         " is NULL or not 2-byte aligned");
    dbuf_status s = check_device(db, "dbuf_pack_grads");
    if (s != DBUF_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t smem = kPackChunk * 2;
    for (int32_t t0 = 0; t0 < db->plan.n; t0 += kMaxPackPtrs) {
        const int32_t t1 = std::min<int32_t>(db->plan.n, t0 + kMaxPackPtrs);
        PackPtrs ptrs;
        std::memset(&ptrs, 0, sizeof ptrs);
        for (int32_t i = t0; i < t1; ++i) ptrs.p[i - t0] = static_cast<const uint16_t*>(grads_bf16[i]);
        const int64_t c0 = db->h_chunk_first[t0], c1 = db->h_chunk_first[t1];
        if (c1 <= c0) continue;
        pack_kernel<<<(unsigned)(c1 - c0), kPackThreads, smem, st>>>(ptrs, db->chunks, c0, t0, db->grad,
                                                                      db->plan.bucket, scale, db->status);
        CUDA_TRY(cudaGetLastError(), "dbuf_pack_grads: launch");
    }
    return DBUF_OK;
}

static dbuf_status step_checks(dbuf_t* db, const dbuf_adam_hparams* hp, const char* who) {
    if (!db) return fail(DBUF_EINVAL, std::string(who) + ": db is NULL");
    if (!hp) return fail(DBUF_EINVAL, std::string(who) + ": hp is NULL");
    if (hp->step < 1) return fail(DBUF_EINVAL, std::string(who) + ": step must be >= 1");
    if (!(hp->beta1 >= 0.f && hp->beta1 < 1.f && hp->beta2 >= 0.f && hp->beta2 < 1.f))
        return fail(DBUF_EINVAL, std::string(who) + ": betas must be in [0, 1)");
    return check_device(db, who);
}

extern "C" dbuf_status dbuf_adam8_step(dbuf_t* db, const dbuf_adam_hparams* hp, float grad_scale, void* stream) {
    dbuf_status s = step_checks(db, hp, "dbuf_adam8_step");
    if (s != DBUF_OK) return s;
    if (db->h_tiles.empty()) return DBUF_OK;
    const StepC c = make_step_constants(*hp, grad_scale);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    adam8_step_kernel<<<(unsigned)db->h_tiles.size(), kThreads, 0, st>>>(
        db->tiles, (int64_t)db->h_tiles.size(), db->plan.bucket, db->master, db->param, db->grad, db->mq, db->vq,
        db->scales, db->plan.n_blocks, c, db->status);
    CUDA_TRY(cudaGetLastError(), "dbuf_adam8_step: launch");
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_adam8_step_host(dbuf_t* db, const dbuf_adam_hparams* hp, float grad_scale,
                                            const void* grads_host, void* params_bf16_host, void* stream) {
    dbuf_status s = step_checks(db, hp, "dbuf_adam8_step_host");
    if (s != DBUF_OK) return s;
    if (db->plan.bucket > 0 && (!grads_host || !params_bf16_host))
        return fail(DBUF_EINVAL, "dbuf_adam8_step_host: host buffer is NULL");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t bytes = (size_t)db->plan.bucket * 2;
    if (bytes) CUDA_TRY(cudaMemcpyAsync(db->grad, grads_host, bytes, cudaMemcpyHostToDevice, st),
                        "dbuf_adam8_step_host: copy in");
    s = dbuf_adam8_step(db, hp, grad_scale, stream);
    if (s != DBUF_OK) return s;
    if (bytes) CUDA_TRY(cudaMemcpyAsync(params_bf16_host, db->param, bytes, cudaMemcpyDeviceToHost, st),
                        "dbuf_adam8_step_host: copy out");
    return DBUF_OK;
}

static void* array_of(const dbuf_t* db, dbuf_which w, size_t* esize) {
    switch (w) {
        case DBUF_MASTER_F32: *esize = 4; return db->master;
        case DBUF_PARAM_BF16: *esize = 2; return db->param;
        case DBUF_GRAD_BF16: *esize = 2; return db->grad;
        case DBUF_M_I8: *esize = 1; return db->mq;
        case DBUF_V_U8: *esize = 1; return db->vq;
    }
    return nullptr;
}

extern "C" dbuf_status dbuf_unpack_views(const dbuf_t* db, dbuf_which which, dbuf_view* out) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_unpack_views: db is NULL");
    size_t es = 0;
    char* a = static_cast<char*>(array_of(db, which, &es));
    if (!a) return fail(DBUF_EINVAL, "dbuf_unpack_views: unknown array kind");
    if (db->plan.n > 0 && !out) return fail(DBUF_EINVAL, "dbuf_unpack_views: out is NULL");
    for (int32_t i = 0; i < db->plan.n; ++i)
        out[i] = dbuf_view{a + (size_t)db->plan.offset[i] * es, db->plan.rows[i], db->plan.cols[i], db->plan.offset[i]};
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_bucket(const dbuf_t* db, dbuf_which which, void** ptr, int64_t* elems) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_bucket: db is NULL");
    size_t es = 0;
    void* a = array_of(db, which, &es);
    if (!a) return fail(DBUF_EINVAL, "dbuf_bucket: unknown array kind");
    if (ptr) *ptr = a;
    if (elems) *elems = db->plan.bucket;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_scales(const dbuf_t* db, float** scales, int64_t* n_blocks) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_scales: db is NULL");
    if (scales) *scales = reinterpret_cast<float*>(db->scales);
    if (n_blocks) *n_blocks = db->plan.n_blocks;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_get_device_status(dbuf_t* db, int32_t* code, void* stream) {
    if (!db || !code) return fail(DBUF_EINVAL, "dbuf_get_device_status: NULL argument");
    dbuf_status s = check_device(db, "dbuf_get_device_status");
    if (s != DBUF_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t h = 0;
    CUDA_TRY(cudaMemcpyAsync(&h, db->status, sizeof h, cudaMemcpyDeviceToHost, st), "dbuf_get_device_status");
    CUDA_TRY(cudaStreamSynchronize(st), "dbuf_get_device_status: sync");
    *code = h;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_clear_device_status(dbuf_t* db, void* stream) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_clear_device_status: db is NULL");
    dbuf_status s = check_device(db, "dbuf_clear_device_status");
    if (s != DBUF_OK) return s;
    CUDA_TRY(cudaMemsetAsync(db->status, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)),
             "dbuf_clear_device_status");
    return DBUF_OK;
}

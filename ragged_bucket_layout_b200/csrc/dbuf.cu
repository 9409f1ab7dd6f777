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

constexpr int kThreads = 512;          // threads per CTA of the step kernel
constexpr int kAlign = 16;             // tensor starts are multiples of 16 elements
constexpr int kTile = 4096;            // elements per tile (8 per thread)
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
                const int64_t cap = kTile - (e0 & (kAlign - 1));
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

// Per-step scalars (formed on the host in double, rounded to float once).
// The bias corrections are folded into the step size and eps:
//   (lr/bc1) m / (sqrt(v)/sqrt(bc2) + eps) = step_hat * m / (sqrt(v) + eps_hat).
struct StepC {
    float b1, omb1, b2, omb2, eps_hat, step_hat, decay, gscale;
};

constexpr int kV = 8;  // elements per thread-vector in the step kernel

__device__ __forceinline__ void set_status(int32_t* status, int32_t code) { atomicCAS(status, 0, code); }

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// Code bytes to float without the conversion unit: a byte b placed in the
// low mantissa bits of 2^23 reads as 2^23 + b; subtracting 2^23 is exact.
// int8 codes are stored with the sign bit flipped first (b = code + 128).
__device__ __forceinline__ float ubyte_to_f(uint32_t w, uint32_t sel) {
    return __fsub_rn(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | sel)), 8388608.0f);
}
__device__ __forceinline__ float sbyte_to_f(uint32_t w_flipped, uint32_t sel) {
    return __fsub_rn(__uint_as_float(__byte_perm(w_flipped, 0x4B000000u, 0x7540u | sel)), 8388736.0f);
}

// Round to the nearest integer, ties to even, by adding 1.5*2^23: the sum
// lies where the float spacing is 1, so the addition itself rounds; the
// low byte of the result's bits is the integer's two's-complement low byte.
// Valid for |x| < 2^22; the codes here satisfy |x| <= 255.
__device__ __forceinline__ uint32_t rne_low_bits(float x) { return __float_as_uint(__fadd_rn(x, 12582912.0f)); }

__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// New m and sqrt(v) of one element, every operation rounded on its own.
__device__ __forceinline__ void new_m_r(float graw, float qmf, float qvf, float dqm, float dqv, const StepC& c,
                                        float& m, float& r) {
    const float g = __fmul_rn(graw, c.gscale);
    const float mo = __fmul_rn(qmf, dqm);
    const float so = __fmul_rn(qvf, dqv);
    const float vo = __fmul_rn(so, so);
    m = __fadd_rn(__fmul_rn(c.b1, mo), __fmul_rn(c.omb1, g));
    const float v = __fadd_rn(__fmul_rn(c.b2, vo), __fmul_rn(c.omb2, __fmul_rn(g, g)));
    r = __fsqrt_rn(v);
}

__device__ __forceinline__ float new_p(float p, float m, float r, const StepC& c) {
    const float u = __fdiv_rn(m, __fadd_rn(r, c.eps_hat));
    return __fsub_rn(__fmul_rn(p, c.decay), __fmul_rn(c.step_hat, u));
}

// Inputs of one thread-vector (8 consecutive bucket elements).
struct In8 {
    uint32_t g[4];   // bf16 pairs
    float p[8];
    uint32_t mq[2];  // int8 codes with the sign bit flipped
    uint32_t vq[2];  // uint8 codes
};

// Load elements [vb, vb+8); when !FULL only those in [lo, hi) are read and
// the rest are zero.
template <bool FULL>
__device__ __forceinline__ void load8(In8& x, int64_t vb, int64_t lo, int64_t hi, bool want_p, const float* master,
                                      const uint16_t* grad, const int8_t* mq, const uint8_t* vq) {
    if (FULL) {
        const uint4 g = __ldg(reinterpret_cast<const uint4*>(grad + vb));
        x.g[0] = g.x; x.g[1] = g.y; x.g[2] = g.z; x.g[3] = g.w;
        const uint2 a = *reinterpret_cast<const uint2*>(mq + vb);
        const uint2 b = *reinterpret_cast<const uint2*>(vq + vb);
        x.mq[0] = a.x ^ 0x80808080u; x.mq[1] = a.y ^ 0x80808080u;
        x.vq[0] = b.x; x.vq[1] = b.y;
        if (want_p) {
            const float4 p0 = __ldcs(reinterpret_cast<const float4*>(master + vb));
            const float4 p1 = __ldcs(reinterpret_cast<const float4*>(master + vb) + 1);
            x.p[0] = p0.x; x.p[1] = p0.y; x.p[2] = p0.z; x.p[3] = p0.w;
            x.p[4] = p1.x; x.p[5] = p1.y; x.p[6] = p1.z; x.p[7] = p1.w;
        }
    } else {
        uint32_t g[4] = {0, 0, 0, 0}, a[2] = {0, 0}, b[2] = {0, 0};
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            const int64_t e = vb + i;
            const bool in = (e >= lo && e < hi);
            x.p[i] = (in && want_p) ? master[e] : 0.f;
            if (in) {
                g[i >> 1] |= (uint32_t)grad[e] << (16 * (i & 1));
                a[i >> 2] |= (uint32_t)(uint8_t)mq[e] << (8 * (i & 3));
                b[i >> 2] |= (uint32_t)vq[e] << (8 * (i & 3));
            }
        }
        x.g[0] = g[0]; x.g[1] = g[1]; x.g[2] = g[2]; x.g[3] = g[3];
        x.mq[0] = a[0] ^ 0x80808080u; x.mq[1] = a[1] ^ 0x80808080u;
        x.vq[0] = b[0]; x.vq[1] = b[1];
    }
}

__device__ __forceinline__ float g_of(const In8& x, int i) {
    const uint32_t w = x.g[i >> 1];
    return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
}

// Update 8 elements; dq* are per element (equal when the vector lies in one block).
__device__ __forceinline__ void update8(In8& x, const float* dqm, const float* dqv, const StepC& c, float* m,
                                        float* r) {
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        new_m_r(g_of(x, i), sbyte_to_f(x.mq[i >> 2], i & 3), ubyte_to_f(x.vq[i >> 2], i & 3), dqm[i], dqv[i], c, m[i],
                r[i]);
        x.p[i] = new_p(x.p[i], m[i], r[i], c);
    }
}

template <bool FULL>
__device__ __forceinline__ void store_p8(const float* p, int64_t vb, int64_t lo, int64_t hi, float* master,
                                         uint16_t* param) {
    const uint4 h = make_uint4(bf16x2_bits(p[0], p[1]), bf16x2_bits(p[2], p[3]), bf16x2_bits(p[4], p[5]),
                               bf16x2_bits(p[6], p[7]));
    if (FULL) {
        __stcs(reinterpret_cast<float4*>(master + vb), make_float4(p[0], p[1], p[2], p[3]));
        __stcs(reinterpret_cast<float4*>(master + vb) + 1, make_float4(p[4], p[5], p[6], p[7]));
        __stcs(reinterpret_cast<uint4*>(param + vb), h);
    } else {
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            const int64_t e = vb + i;
            if (e >= lo && e < hi) {
                master[e] = p[i];
                param[e] = (uint16_t)(hw[i >> 1] >> (16 * (i & 1)));
            }
        }
    }
}

// Codes of 8 elements from m, r and the per-element quotients 127/absmax,
// 255/absmax.  |m*qm| <= 127 and 0 <= r*qv <= 255 hold by construction
// (absmax over the same values), so rounding never needs a clamp.
template <bool FULL>
__device__ __forceinline__ void store_codes8(const float* m, const float* r, const float* qm, const float* qv,
                                             int64_t vb, int64_t lo, int64_t hi, int8_t* mq, uint8_t* vq) {
    uint32_t bm[kV], bv[kV];
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        bm[i] = rne_low_bits(__fmul_rn(m[i], qm[i]));
        bv[i] = rne_low_bits(__fmul_rn(r[i], qv[i]));
    }
    const uint2 cm = make_uint2(pack_low_bytes(bm[0], bm[1], bm[2], bm[3]), pack_low_bytes(bm[4], bm[5], bm[6], bm[7]));
    const uint2 cv = make_uint2(pack_low_bytes(bv[0], bv[1], bv[2], bv[3]), pack_low_bytes(bv[4], bv[5], bv[6], bv[7]));
    if (FULL) {
        __stcs(reinterpret_cast<uint2*>(mq + vb), cm);
        __stcs(reinterpret_cast<uint2*>(vq + vb), cv);
    } else {
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            const int64_t e = vb + i;
            if (e >= lo && e < hi) {
                mq[e] = (int8_t)(bm[i] & 0xffu);
                vq[e] = (uint8_t)(bv[i] & 0xffu);
            }
        }
    }
}

// Max over the lanes of a warp that share `key`, where lanes with equal keys
// are contiguous; the first lane of each run ends with the run's maximum.
__device__ __forceinline__ bool segmented_max(int key, float& a, float& b) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int ok = __shfl_down_sync(0xffffffffu, key, d);
        const float oa = __shfl_down_sync(0xffffffffu, a, d);
        const float ob = __shfl_down_sync(0xffffffffu, b, d);
        if (lane + d < 32 && ok == key) {
            a = fmaxf(a, oa);
            b = fmaxf(b, ob);
        }
    }
    const int prev = __shfl_up_sync(0xffffffffu, key, 1);
    return (lane == 0) || (prev != key);
}

__device__ __forceinline__ void warp_max2(float& a, float& b) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, d));
        b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, d));
    }
}

// Phase 1 of a whole-block tile for a thread-vector that lies in one block:
// load, update, write the weights.  No barrier in here: FULL and partial
// vectors of one warp run different instances of this function.
template <bool FULL>
__device__ __forceinline__ void phase1_one(int64_t vb, int64_t lo, int64_t hi, float dqm, float dqv, float* master,
                                           uint16_t* param, const uint16_t* grad, const int8_t* mq,
                                           const uint8_t* vq, const StepC& c, float* m, float* r) {
    In8 x;
    load8<FULL>(x, vb, lo, hi, true, master, grad, mq, vq);
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        new_m_r(g_of(x, i), sbyte_to_f(x.mq[i >> 2], i & 3), ubyte_to_f(x.vq[i >> 2], i & 3), dqm, dqv, c, m[i],
                r[i]);
        x.p[i] = new_p(x.p[i], m[i], r[i], c);
    }
    store_p8<FULL>(x.p, vb, lo, hi, master, param);
}

// The same for a vector that spans several blocks (blocks shorter than 8
// elements, or off the 8-element grid): per-element block numbers.
__device__ __noinline__ void phase1_mixed(int64_t vb, int64_t lo, int64_t hi, uint32_t b, int bf, float* master,
                                          uint16_t* param, const uint16_t* grad, const int8_t* mq,
                                          const uint8_t* vq, const StepC& c, const float* s_dqm,
                                          const float* s_dqv, uint32_t* s_am, uint32_t* s_ar, float* m,
                                          float* r) {
    In8 x;
    load8<false>(x, vb, lo, hi, true, master, grad, mq, vq);
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        const int64_t e = vb + i;
        const int blk = (e < lo || e >= hi) ? bf : (int)((uint32_t)(e - lo) / b);
        new_m_r(g_of(x, i), sbyte_to_f(x.mq[i >> 2], i & 3), ubyte_to_f(x.vq[i >> 2], i & 3), s_dqm[blk],
                s_dqv[blk], c, m[i], r[i]);
        x.p[i] = new_p(x.p[i], m[i], r[i], c);
        atomicMax(&s_am[blk], __float_as_uint(fabsf(m[i])));
        atomicMax(&s_ar[blk], __float_as_uint(r[i]));
    }
    store_p8<false>(x.p, vb, lo, hi, master, param);
}

__device__ __noinline__ void codes_mixed(int64_t vb, int64_t lo, int64_t hi, uint32_t b, int bf, const float* s_qm,
                                         const float* s_qv, const float* m, const float* r, int8_t* mq,
                                         uint8_t* vq) {
    float qm[kV], qv[kV];
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        const int64_t e = vb + i;
        const int blk = (e < lo || e >= hi) ? bf : (int)((uint32_t)(e - lo) / b);
        qm[i] = s_qm[blk];
        qv[i] = s_qv[blk];
    }
    store_codes8<false>(m, r, qm, qv, vb, lo, hi, mq, vq);
}

template <bool FULL>
__device__ __forceinline__ void codes_one(int64_t vb, int64_t lo, int64_t hi, float qm1, float qv1, const float* m,
                                          const float* r, int8_t* mq, uint8_t* vq) {
    float qm[kV], qv[kV];
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        qm[i] = qm1;
        qv[i] = qv1;
    }
    store_codes8<FULL>(m, r, qm, qv, vb, lo, hi, mq, vq);
}

// Up to 256 whole blocks of one tensor.  Non-negative floats order like
// their bit patterns, so block maxima are kept as unsigned integers for
// atomicMax in shared memory.
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
    const int64_t vb = (t.e0 & ~int64_t(kAlign - 1)) + (int64_t)kV * tid;
    const int64_t elo = max(vb, lo), ehi = min(vb + kV, hi);
    const bool any = elo < ehi;
    const bool full = (vb >= lo) && (vb + kV <= hi);
    const uint32_t b = (uint32_t)t.b;
    const bool single = t.nblk == 1;
    // block of the first and last element of this vector
    const int bf = any ? (single ? 0 : (int)((uint32_t)(elo - lo) / b)) : -1;
    const int bl = any ? (single ? 0 : (int)((uint32_t)(ehi - 1 - lo) / b)) : -1;
    const bool one = (bf == bl);
    float m[kV], r[kV];        // registers (fast path)
    float mx[kV], rx[kV];      // the mixed path's copies (passed by address)
    float am = 0.f, ar = 0.f;  // elements outside the tile have m = r = 0
    if (any && one) {
        const float dqm = s_dqm[bf], dqv = s_dqv[bf];
        if (full)
            phase1_one<true>(vb, lo, hi, dqm, dqv, master, param, grad, mq, vq, c, m, r);
        else
            phase1_one<false>(vb, lo, hi, dqm, dqv, master, param, grad, mq, vq, c, m, r);
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            am = fmaxf(am, fabsf(m[i]));
            ar = fmaxf(ar, r[i]);
        }
    } else if (any) {
        phase1_mixed(vb, lo, hi, b, bf, master, param, grad, mq, vq, c, s_dqm, s_dqv, s_am, s_ar, mx, rx);
    }
    if (single) {
        warp_max2(am, ar);
        if ((tid & 31) == 0) {
            atomicMax(&s_am[0], __float_as_uint(am));
            atomicMax(&s_ar[0], __float_as_uint(ar));
        }
    } else {
        const int key = (any && one) ? bf : -1;
        if (segmented_max(key, am, ar) && key >= 0) {
            atomicMax(&s_am[key], __float_as_uint(am));
            atomicMax(&s_ar[key], __float_as_uint(ar));
        }
    }
    __syncthreads();
    if (tid < t.nblk) {
        const float AMm = __uint_as_float(s_am[tid]), AMr = __uint_as_float(s_ar[tid]);
        s_qm[tid] = AMm > 0.f ? __fdiv_rn(127.f, AMm) : 0.f;
        s_qv[tid] = AMr > 0.f ? __fdiv_rn(255.f, AMr) : 0.f;
        scales[t.blk0 + tid] = make_float2(AMm, AMr);
    }
    __syncthreads();
    if (any && one) {
        const float qm = s_qm[bf], qv = s_qv[bf];
        if (full)
            codes_one<true>(vb, lo, hi, qm, qv, m, r, mq, vq);
        else
            codes_one<false>(vb, lo, hi, qm, qv, m, r, mq, vq);
    } else if (any) {
        codes_mixed(vb, lo, hi, b, bf, s_qm, s_qv, mx, rx, mq, vq);
    }
}

template <bool FULL>
__device__ __forceinline__ void large_pass1_vec(int64_t vb, int64_t lo, int64_t hi, float dqm1, float dqv1,
                                                float* master, uint16_t* param, const uint16_t* grad,
                                                const int8_t* mq, const uint8_t* vq, const StepC& c, float& am,
                                                float& ar) {
    In8 x;
    float dqm[kV], dqv[kV], m[kV], r[kV];
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        dqm[i] = dqm1;
        dqv[i] = dqv1;
    }
    load8<FULL>(x, vb, lo, hi, true, master, grad, mq, vq);
    update8(x, dqm, dqv, c, m, r);
    store_p8<FULL>(x.p, vb, lo, hi, master, param);
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        am = fmaxf(am, fabsf(m[i]));
        ar = fmaxf(ar, r[i]);
    }
}

template <bool FULL>
__device__ __forceinline__ void large_pass2_vec(int64_t vb, int64_t lo, int64_t hi, float dqm1, float dqv1,
                                                float qm1, float qv1, const uint16_t* grad, int8_t* mq, uint8_t* vq,
                                                const StepC& c) {
    In8 x;
    float m[kV], r[kV], qm[kV], qv[kV];
    load8<FULL>(x, vb, lo, hi, false, nullptr, grad, mq, vq);
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        new_m_r(g_of(x, i), sbyte_to_f(x.mq[i >> 2], i & 3), ubyte_to_f(x.vq[i >> 2], i & 3), dqm1, dqv1, c, m[i],
                r[i]);
        qm[i] = qm1;
        qv[i] = qv1;
    }
    store_codes8<FULL>(m, r, qm, qv, vb, lo, hi, mq, vq);
}

__device__ void large_block(const Tile& t, float* master, uint16_t* param, const uint16_t* grad, int8_t* mq,
                            uint8_t* vq, float2* scales, const StepC& c) {
    __shared__ float s_red[2][kThreads / 32];
    __shared__ float s_q[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float2 sc = scales[t.blk0];
    const float dqm = __fdiv_rn(sc.x, 127.f), dqv = __fdiv_rn(sc.y, 255.f);
    const int64_t lo = t.e0, hi = t.e0 + t.n;
    const int64_t a0 = t.e0 & ~int64_t(kAlign - 1);

    // Pass 1: full update, weights written, absmax accumulated.
    float am = 0.f, ar = 0.f;
    for (int64_t vb = a0 + (int64_t)kV * tid; vb < hi; vb += kTile) {
        if (vb >= lo && vb + kV <= hi)
            large_pass1_vec<true>(vb, lo, hi, dqm, dqv, master, param, grad, mq, vq, c, am, ar);
        else
            large_pass1_vec<false>(vb, lo, hi, dqm, dqv, master, param, grad, mq, vq, c, am, ar);
    }
    warp_max2(am, ar);
    if (lane == 0) {
        s_red[0][warp] = am;
        s_red[1][warp] = ar;
    }
    __syncthreads();
    if (tid == 0) {
        float a = 0.f, b = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) {
            a = fmaxf(a, s_red[0][w]);
            b = fmaxf(b, s_red[1][w]);
        }
        s_q[0] = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
        s_q[1] = b > 0.f ? __fdiv_rn(255.f, b) : 0.f;
        scales[t.blk0] = make_float2(a, b);
    }
    __syncthreads();
    const float qm = s_q[0], qv = s_q[1];

    // Pass 2: recompute m and sqrt(v) from the unchanged grad and old codes.
    for (int64_t vb = a0 + (int64_t)kV * tid; vb < hi; vb += kTile) {
        if (vb >= lo && vb + kV <= hi)
            large_pass2_vec<true>(vb, lo, hi, dqm, dqv, qm, qv, grad, mq, vq, c);
        else
            large_pass2_vec<false>(vb, lo, hi, dqm, dqv, qm, qv, grad, mq, vq, c);
    }
}

__device__ void zero_tile(const Tile& t, uint16_t* param) {
    const int64_t lo = t.e0, hi = t.e0 + t.n;
    const int64_t a0 = t.e0 & ~int64_t(kAlign - 1);
    for (int64_t vb = a0 + (int64_t)kV * threadIdx.x; vb < hi; vb += kTile) {
        if (vb >= lo && vb + kV <= hi) {
            __stcs(reinterpret_cast<uint4*>(param + vb), make_uint4(0, 0, 0, 0));
        } else {
            for (int i = 0; i < kV; ++i)
                if (vb + i >= lo && vb + i < hi) param[vb + i] = 0;
        }
    }
}

__global__ void __launch_bounds__(kThreads, 2) adam8_step_kernel(const Tile* __restrict__ tiles, int64_t n_tiles,
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
        (t.kind == TILE_WHOLE && (t.b <= 0 || t.nblk > kMaxBlk || (t.e0 & (kAlign - 1)) + t.n > kTile))) {
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
    const double B1 = hp.beta1, B2 = hp.beta2, lr = hp.lr, wd = hp.weight_decay, eps = hp.eps;
    const double t = (double)hp.step;
    const double bc1 = 1.0 - std::pow(B1, t);
    const double sq2 = std::sqrt(1.0 - std::pow(B2, t));
    StepC c;
    c.b1 = (float)B1;
    c.omb1 = (float)(1.0 - B1);
    c.b2 = (float)B2;
    c.omb2 = (float)(1.0 - B2);
    c.eps_hat = (float)(eps * sq2);
    c.step_hat = (float)(lr * sq2 / bc1);
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
    if (plan->align % kAlign != 0)
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

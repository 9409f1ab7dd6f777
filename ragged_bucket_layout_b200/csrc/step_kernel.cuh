// Fused block-wise 8-bit Adam step over a whole ragged bucket (sm_100a).
//
// veScale-FSDP (8-bit Adam case study, paper Sec. 6.3; DBuffer group
// operations, Sec. 5): the quantisation blocks are aligned with the shards,
// so every block is updated and requantised on its own, and the whole
// bucket goes through one grouped launch instead of one launch per tensor.
//
// Persistent kernel, one CTA per slot (three per SM): 8 consumer warps and
// one producer warp.  The producer walks the CTA's share of the work table
// (entries blockIdx.x, blockIdx.x + gridDim.x, ...) and streams each tile's
// inputs (bf16 grad, fp32 master, int8/uint8 codes, per-block scales) into a
// 2-stage shared-memory ring with bulk copies (TMA, cp.async.bulk), so the
// loads of the next tiles are in flight while the consumers compute and wait
// at barriers.  Consumers read a stage (16 elements per thread, as two
// 8-element vectors), write weights and the bf16 copy straight to global
// memory, put the new m and sqrt(v) back into their own bytes of the stage,
// reduce each block's absmax, then read m and sqrt(v) back and write the
// codes.  A LARGE block (longer than a tile) is streamed twice: pass 1
// updates the weights and finds the absmax; pass 2 reloads grad and the old
// codes (recently read, so mostly from L2) and recomputes m and sqrt(v)
// bit-identically to quantise them.
//
// Waits on copies are bounded (2 s); a time-out sets status 1 and the CTA
// drains its own copies before leaving.  One elected consumer thread waits
// and a named barrier hands the outcome to all consumers, so they agree.
#pragma once

#include <cuda_bf16.h>

#include "fastmath.cuh"
#include "tables.h"
#include "tma.cuh"

namespace dbuf_k {

// Per-step scalars (formed on the host in double, rounded to float once).
// The bias corrections are folded into the step size and eps:
//   (lr/bc1) m / (sqrt(v)/sqrt(bc2) + eps) = step_hat * m / (sqrt(v) + eps_hat).
struct StepC {
    float b1, omb1, b2, omb2, eps_hat, step_hat, decay, gscale;
};

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;       // 256 threads
constexpr int kStepThreads = kConsumers + 32;         // + one producer warp
#ifndef DBUF_STEP_STAGES
#define DBUF_STEP_STAGES 2  // shared-memory ring depth
#endif
#ifndef DBUF_STEP_MIN_CTAS
#define DBUF_STEP_MIN_CTAS 3  // CTAs per SM the register budget is sized for
#endif
constexpr int kStages = DBUF_STEP_STAGES;
constexpr int kV = 8;                                 // elements per thread-vector
constexpr int kSub = kTile / (kConsumers * kV);       // vectors per thread per tile (2)
constexpr int kOffG = 0;                              // bf16 grad
constexpr int kOffP = kOffG + kTile * 2;              // fp32 master
constexpr int kOffMQ = kOffP + kTile * 4;             // int8 codes of m
constexpr int kOffVQ = kOffMQ + kTile;                // uint8 codes of sqrt(v)
constexpr int kOffS = kOffVQ + kTile;                 // float2 scales (<= 256 entries)
constexpr int kStageBytes = kOffS + 256 * 8;          // 34816
constexpr int kStepSmem = kStages * kStageBytes;
constexpr uint32_t kBarCons = 1;                      // named barrier of the consumers
static_assert(kSub * kConsumers * kV == kTile, "tile split");
static_assert(kMaxBlk + 2 <= 256, "scale copy fits its stage slot");

struct StepShared {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint32_t am[256], ar[256];  // block absmax as float bits
    float dqm[256], dqv[256];   // dequantisation steps of the old codes
    float qm[256], qv[256];     // quantisation factors of the new codes
    float red[2][kConsumerWarps];
    uint32_t am1[2], ar1[2];    // single-block tiles: absmax, double-buffered by tile parity
    int32_t go[2];
};

// ---------------------------------------------------------------- arithmetic

// Code bytes to float without the conversion unit: byte b in the low
// mantissa bits of 2^23 reads as 2^23 + b; subtracting 2^23 is exact.  int8
// codes have their sign bit flipped first (b = code + 128).
__device__ __forceinline__ float ubyte_to_f(uint32_t w, uint32_t sel) {
    return __fsub_rn(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | sel)), 8388608.0f);
}
__device__ __forceinline__ float sbyte_to_f(uint32_t w_flipped, uint32_t sel) {
    return __fsub_rn(__uint_as_float(__byte_perm(w_flipped, 0x4B000000u, 0x7540u | sel)), 8388736.0f);
}

// Round to the nearest integer, ties to even, by adding 1.5*2^23: the sum
// lies where the float spacing is 1, so the addition itself rounds, and the
// low byte of the sum's bits is the integer's two's-complement low byte.
// Valid for |x| < 2^22; codes here have |x| <= 255.
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

// The same arithmetic on two elements at once with the paired fp32
// instructions of sm_100 (mul/add .f32x2, written as PTX with .rn): each
// component is rounded exactly as the scalar instruction.  A paired add
// whose operands are paired products is fused into one FMA by the
// assembler (measured: about a third of results move by one ulp), so every
// add that consumes a product stays scalar (__fadd_rn/__fsub_rn are never
// fused); only adds of non-products use add2.
__device__ __forceinline__ float2 dup(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
// Scalar sums / differences of two paired products, component by component.
__device__ __forceinline__ float2 sum_of(float2 a, float2 b) {
    return make_float2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
}
__device__ __forceinline__ float2 diff_of(float2 a, float2 b) {
    return make_float2(__fsub_rn(a.x, b.x), __fsub_rn(a.y, b.y));
}

// Code bytes i, i+1 of a word as two exact floats (see ubyte_to_f).
__device__ __forceinline__ float2 ubytes_to_f2(uint32_t w, uint32_t i, float bias) {
    const float2 x = make_float2(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | i)),
                                 __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | (i + 1))));
    return add2(x, dup(-bias));
}

struct StepC2 {
    float2 b1, omb1, b2, omb2, eps_hat, step_hat, decay, gscale;
};


// New m and v for elements (2j, 2j+1) of a vector (sqrt(v) taken per vector).
__device__ __forceinline__ void new_m_v2(float2 graw, float2 qmf, float2 qvf, float2 dqm, float2 dqv,
                                         const StepC2& c, float2 gs, float2& m, float2& v) {
    const float2 g = mul2(graw, gs);
    const float2 mo = mul2(qmf, dqm);
    const float2 so = mul2(qvf, dqv);
    const float2 vo = mul2(so, so);
    m = sum_of(mul2(c.b1, mo), mul2(c.omb1, g));
    v = sum_of(mul2(c.b2, vo), mul2(c.omb2, mul2(g, g)));
}

// Correctly rounded sqrt of the 4 pairs of a vector: the fast sequence
// when every v is in its checked range (the normal case), else IEEE sqrt.
__device__ __forceinline__ void sqrt_vec(const float2* v, float2* r) {
    uint32_t lo = 0xffffffffu;
#pragma unroll
    for (int j = 0; j < kV / 2; ++j) lo = min(lo, min(__float_as_uint(v[j].x), __float_as_uint(v[j].y)));
    if (lo >= kSqrtFastMinBits) {
#pragma unroll
        for (int j = 0; j < kV / 2; ++j) r[j] = sqrt2_fast(v[j]);
    } else {
#pragma unroll
        for (int j = 0; j < kV / 2; ++j) r[j] = make_float2(__fsqrt_rn(v[j].x), __fsqrt_rn(v[j].y));
    }
}

template <bool FAST>
__device__ __forceinline__ float2 new_p2(float2 p, float2 m, float2 r, const StepC2& c) {
    const float2 d = sum_of(r, c.eps_hat);  // r ends a square-root sequence: keep the add scalar
    const float2 u = FAST ? div2_fast(m, d) : make_float2(__fdiv_rn(m.x, d.x), __fdiv_rn(m.y, d.y));
    return diff_of(mul2(p, c.decay), mul2(c.step_hat, u));
}

// ------------------------------------------------------------ vector I/O
//
// Thread-vector = 8 consecutive elements at local index li (a multiple of 8)
// of a stage.  Its bytes in the stage: grad [2li, 2li+16), master
// [4li, 4li+32), codes [li, li+8) twice.  After phase 1 the thread's new m
// goes to its master bytes and its new sqrt(v) to its grad (4 values) and
// code bytes (2 + 2 values): 32 + 32 bytes that no other thread touches.
// The two 16-byte halves of a thread's master bytes are taken in the order
// h, 1-h with h = bit 2 of the thread index, so each group of 8 threads
// covers all 32 banks once per access.

struct In8 {
    uint32_t g[4];   // bf16 pairs
    float p[8];
    uint32_t mq[2];  // int8 codes, sign bits flipped
    uint32_t vq[2];  // uint8 codes
};

__device__ __forceinline__ float g_of(const In8& x, int i) {
    const uint32_t w = x.g[i >> 1];
    return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
}

__device__ __forceinline__ int half_order() { return (threadIdx.x >> 2) & 1; }

__device__ __forceinline__ void lds_f8(const unsigned char* base, float* v) {
    const int h = half_order();
    const float4 a = *reinterpret_cast<const float4*>(base + 16 * h);
    const float4 b = *reinterpret_cast<const float4*>(base + 16 * (1 - h));
    const float4 lo = h ? b : a, hi = h ? a : b;
    v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
    v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
}

__device__ __forceinline__ void sts_f8(unsigned char* base, const float* v) {
    const int h = half_order();
    const float4 lo = make_float4(v[0], v[1], v[2], v[3]), hi = make_float4(v[4], v[5], v[6], v[7]);
    *reinterpret_cast<float4*>(base + 16 * h) = h ? hi : lo;
    *reinterpret_cast<float4*>(base + 16 * (1 - h)) = h ? lo : hi;
}

// When !FULL only local elements in [lo, hi) are taken; the rest read as zero.
template <bool FULL>
__device__ __forceinline__ void load8(In8& x, const unsigned char* st, int li, int lo, int hi, bool want_p) {
    if (FULL) {
        const uint4 g = *reinterpret_cast<const uint4*>(st + kOffG + 2 * li);
        x.g[0] = g.x; x.g[1] = g.y; x.g[2] = g.z; x.g[3] = g.w;
        const uint2 a = *reinterpret_cast<const uint2*>(st + kOffMQ + li);
        const uint2 b = *reinterpret_cast<const uint2*>(st + kOffVQ + li);
        x.mq[0] = a.x ^ 0x80808080u; x.mq[1] = a.y ^ 0x80808080u;
        x.vq[0] = b.x; x.vq[1] = b.y;
        if (want_p) lds_f8(st + kOffP + 4 * li, x.p);
    } else {
        const uint16_t* g = reinterpret_cast<const uint16_t*>(st + kOffG);
        const float* p = reinterpret_cast<const float*>(st + kOffP);
        uint32_t gw[4] = {0, 0, 0, 0}, aw[2] = {0, 0}, bw[2] = {0, 0};
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            const int e = li + i;
            const bool in = (e >= lo && e < hi);
            x.p[i] = (in && want_p) ? p[e] : 0.f;
            if (in) {
                gw[i >> 1] |= (uint32_t)g[e] << (16 * (i & 1));
                aw[i >> 2] |= (uint32_t)st[kOffMQ + e] << (8 * (i & 3));
                bw[i >> 2] |= (uint32_t)st[kOffVQ + e] << (8 * (i & 3));
            }
        }
        x.g[0] = gw[0]; x.g[1] = gw[1]; x.g[2] = gw[2]; x.g[3] = gw[3];
        x.mq[0] = aw[0] ^ 0x80808080u; x.mq[1] = aw[1] ^ 0x80808080u;
        x.vq[0] = bw[0]; x.vq[1] = bw[1];
    }
}

__device__ __forceinline__ void stash_mr(unsigned char* st, int li, const float* m, const float* r) {
    sts_f8(st + kOffP + 4 * li, m);
    *reinterpret_cast<uint4*>(st + kOffG + 2 * li) =
        make_uint4(__float_as_uint(r[0]), __float_as_uint(r[1]), __float_as_uint(r[2]), __float_as_uint(r[3]));
    *reinterpret_cast<uint2*>(st + kOffMQ + li) = make_uint2(__float_as_uint(r[4]), __float_as_uint(r[5]));
    *reinterpret_cast<uint2*>(st + kOffVQ + li) = make_uint2(__float_as_uint(r[6]), __float_as_uint(r[7]));
}

__device__ __forceinline__ void unstash_mr(const unsigned char* st, int li, float* m, float* r) {
    lds_f8(st + kOffP + 4 * li, m);
    const uint4 a = *reinterpret_cast<const uint4*>(st + kOffG + 2 * li);
    const uint2 b = *reinterpret_cast<const uint2*>(st + kOffMQ + li);
    const uint2 d = *reinterpret_cast<const uint2*>(st + kOffVQ + li);
    r[0] = __uint_as_float(a.x); r[1] = __uint_as_float(a.y); r[2] = __uint_as_float(a.z); r[3] = __uint_as_float(a.w);
    r[4] = __uint_as_float(b.x); r[5] = __uint_as_float(b.y);
    r[6] = __uint_as_float(d.x); r[7] = __uint_as_float(d.y);
}

// Global pointers shifted to a window's first element, so the stores take
// 32-bit local indices.
struct Out {
    float* master;
    uint16_t* param;
    int8_t* mq;
    uint8_t* vq;
};

template <bool FULL>
__device__ __forceinline__ void store_p8(const float* p, int li, int lo, int hi, const Out& o) {
    const uint4 h = make_uint4(bf16x2_bits(p[0], p[1]), bf16x2_bits(p[2], p[3]), bf16x2_bits(p[4], p[5]),
                               bf16x2_bits(p[6], p[7]));
    if (FULL) {
        __stcs(reinterpret_cast<float4*>(o.master + li), make_float4(p[0], p[1], p[2], p[3]));
        __stcs(reinterpret_cast<float4*>(o.master + li) + 1, make_float4(p[4], p[5], p[6], p[7]));
        __stcs(reinterpret_cast<uint4*>(o.param + li), h);
    } else {
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            const int e = li + i;
            if (e >= lo && e < hi) {
                o.master[e] = p[i];
                o.param[e] = (uint16_t)(hw[i >> 1] >> (16 * (i & 1)));
            }
        }
    }
}

// Codes of 8 elements.  |m*qm| <= 127 and 0 <= r*qv <= 255 hold by
// construction (qm = 127/max|m| over the same values), so no clamp is needed.
template <bool FULL>
__device__ __forceinline__ void store_codes8(const float* m, const float* r, const float* qm, const float* qv, int li,
                                             int lo, int hi, const Out& o) {
    uint32_t bm[kV], bv[kV];
    const float2 magic = dup(12582912.0f);  // 1.5 * 2^23, see rne_low_bits
#pragma unroll
    for (int j = 0; j < kV / 2; ++j) {
        const float2 a = sum_of(mul2(make_float2(m[2 * j], m[2 * j + 1]), make_float2(qm[2 * j], qm[2 * j + 1])), magic);
        const float2 b = sum_of(mul2(make_float2(r[2 * j], r[2 * j + 1]), make_float2(qv[2 * j], qv[2 * j + 1])), magic);
        bm[2 * j] = __float_as_uint(a.x);
        bm[2 * j + 1] = __float_as_uint(a.y);
        bv[2 * j] = __float_as_uint(b.x);
        bv[2 * j + 1] = __float_as_uint(b.y);
    }
    if (FULL) {
        __stcs(reinterpret_cast<uint2*>(o.mq + li),
               make_uint2(pack_low_bytes(bm[0], bm[1], bm[2], bm[3]), pack_low_bytes(bm[4], bm[5], bm[6], bm[7])));
        __stcs(reinterpret_cast<uint2*>(o.vq + li),
               make_uint2(pack_low_bytes(bv[0], bv[1], bv[2], bv[3]), pack_low_bytes(bv[4], bv[5], bv[6], bv[7])));
    } else {
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            const int e = li + i;
            if (e >= lo && e < hi) {
                o.mq[e] = (int8_t)(bm[i] & 0xffu);
                o.vq[e] = (uint8_t)(bv[i] & 0xffu);
            }
        }
    }
}

// New m and sqrt(v) of a loaded vector whose elements share dqm/dqv.
__device__ __forceinline__ void mr8(const In8& x, float dqm, float dqv, const StepC2& c, float2 gs, float* m,
                                    float* r) {
    const float2 dqm2 = dup(dqm), dqv2 = dup(dqv);
    float2 mm[kV / 2], vv[kV / 2], rr[kV / 2];
#pragma unroll
    for (int j = 0; j < kV / 2; ++j) {
        const uint32_t w = x.g[j];
        const float2 g = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
        const float2 qmf = ubytes_to_f2(x.mq[j >> 1], 2 * (j & 1), 8388736.0f);
        const float2 qvf = ubytes_to_f2(x.vq[j >> 1], 2 * (j & 1), 8388608.0f);
        new_m_v2(g, qmf, qvf, dqm2, dqv2, c, gs, mm[j], vv[j]);
    }
    sqrt_vec(vv, rr);
#pragma unroll
    for (int j = 0; j < kV / 2; ++j) {
        m[2 * j] = mm[j].x;
        m[2 * j + 1] = mm[j].y;
        r[2 * j] = rr[j].x;
        r[2 * j + 1] = rr[j].y;
    }
}

// Update of one vector whose elements share dqm/dqv (one block); am, ar
// receive the vector's max |m| and max sqrt(v).  The division takes the
// fast sequence when the whole vector lies in its range: d = sqrt(v) + eps
// >= eps >= 2^-60 and sqrt(v) <= 2^64 bound d, and |m| is bounded on both
// sides (a zero m takes the IEEE path).
template <bool FULL>
__device__ __forceinline__ void update8(const unsigned char* st, int li, int lo, int hi, float dqm, float dqv,
                                        const StepC2& c, float2 gs, const Out& o, float* m, float* r, float& am,
                                        float& ar) {
    In8 x;
    load8<FULL>(x, st, li, lo, hi, true);
    mr8(x, dqm, dqv, c, gs, m, r);
    float mn = fabsf(m[0]);
    am = 0.f;
    ar = 0.f;
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        am = fmaxf(am, fabsf(m[i]));
        mn = fminf(mn, fabsf(m[i]));
        ar = fmaxf(ar, r[i]);
    }
    const bool fast = am <= kDivMaxA && mn >= kDivMinA && ar <= 0.5f * kDivMaxD && c.eps_hat.x >= kDivMinD;
    if (fast) {
#pragma unroll
        for (int j = 0; j < kV / 2; ++j) {
            const float2 pn = new_p2<true>(make_float2(x.p[2 * j], x.p[2 * j + 1]),
                                           make_float2(m[2 * j], m[2 * j + 1]), make_float2(r[2 * j], r[2 * j + 1]), c);
            x.p[2 * j] = pn.x;
            x.p[2 * j + 1] = pn.y;
        }
    } else {
#pragma unroll
        for (int j = 0; j < kV / 2; ++j) {
            const float2 pn = new_p2<false>(make_float2(x.p[2 * j], x.p[2 * j + 1]),
                                            make_float2(m[2 * j], m[2 * j + 1]), make_float2(r[2 * j], r[2 * j + 1]), c);
            x.p[2 * j] = pn.x;
            x.p[2 * j + 1] = pn.y;
        }
    }
    store_p8<FULL>(x.p, li, lo, hi, o);
}

// ------------------------------------------------------------- reductions

// Max over lanes sharing `key` (equal keys are contiguous lanes); true on the
// first lane of each run, which holds the run's maximum.
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

// Fold (a, b) of every lane into block `key` of shared memory (key < 0: no
// contribution).  One atomic per warp when the whole warp is in one block.
__device__ __forceinline__ void block_max_to_smem(int key, float a, float b, StepShared& sh) {
    const int k0 = __shfl_sync(0xffffffffu, key, 0);
    if (__all_sync(0xffffffffu, key == k0)) {
        warp_max2(a, b);
        if ((threadIdx.x & 31) == 0 && k0 >= 0) {
            atomicMax(&sh.am[k0], __float_as_uint(a));
            atomicMax(&sh.ar[k0], __float_as_uint(b));
        }
    } else if (segmented_max(key, a, b) && key >= 0) {
        atomicMax(&sh.am[key], __float_as_uint(a));
        atomicMax(&sh.ar[key], __float_as_uint(b));
    }
}

// ------------------------------------------------------------ pipeline

__device__ __forceinline__ bool strip_ok(const Tile& t, int64_t bucket, int64_t n_blocks) {
    const int64_t C = t.b, W = t.magic;
    if (C < 16 || (C & 15) || (t.n & 15) || t.n > kTile || t.n > C || t.nblk < 1 || (t.e0 & (kAlign - 1))) return false;
    if (W < 16 || W > kTile || (W & (W - 1))) return false;
    if (t.e0 + (int64_t)(t.nblk - 1) * C + t.n > bucket) return false;
    const int64_t G = (t.n + W - 1) / W;
    return G <= kMaxStripTiles && t.blk0 >= 0 && t.blk0 + G <= n_blocks;
}

__device__ __forceinline__ bool tile_ok(const Tile& t, int64_t bucket, int64_t n_blocks) {
    if (t.e0 < 0 || t.n <= 0 || t.e0 + t.n > bucket) return false;
    if (t.kind == TILE_ZERO) return true;
    if (t.kind == TILE_STRIP) return strip_ok(t, bucket, n_blocks);
    if (t.blk0 < 0 || t.nblk < 1 || t.blk0 + t.nblk > n_blocks) return false;
    if (t.kind == TILE_WHOLE) return t.b > 0 && t.nblk <= kMaxBlk && (t.e0 & (kAlign - 1)) + t.n <= kTile;
    return t.kind == TILE_LARGE && t.nblk == 1;
}

__device__ __forceinline__ int64_t large_chunks(const Tile& t) {
    const int64_t a0 = t.e0 & ~int64_t(kAlign - 1);
    return (t.e0 + t.n - a0 + kTile - 1) / kTile;
}

// Chunking of a STRIP entry: rows per chunk, and chunks per pass.
__device__ __forceinline__ int strip_rows_per_chunk(const Tile& t) { return t.b <= kTile ? kTile / t.b : 1; }
__device__ __forceinline__ int strip_chunks(const Tile& t) {
    const int rpc = strip_rows_per_chunk(t);
    return (t.nblk + rpc - 1) / rpc;
}
// First element and length of chunk ch (both multiples of 16).
__device__ __forceinline__ void strip_chunk(const Tile& t, int ch, int64_t& w0, int& len) {
    const int rpc = strip_rows_per_chunk(t);
    const int rows = min(rpc, t.nblk - ch * rpc);
    w0 = t.e0 + (int64_t)ch * rpc * t.b;
    len = t.b <= kTile ? rows * t.b : (int)t.n;
}

// Consumers: wait until stage use k has landed.  Thread 0 waits (bounded),
// the named barrier hands its verdict to every consumer.
__device__ __forceinline__ bool wait_stage(StepShared& sh, uint32_t k, int32_t* status) {
    if (threadIdx.x == 0) {
        const bool ok = mbar_wait_bounded(&sh.full[k % kStages], (k / kStages) & 1u);
        sh.go[k & 1u] = ok ? 1 : 0;
        if (!ok) set_status(status, 1);
    }
    named_sync(kBarCons, kConsumers);
    return sh.go[k & 1u] != 0;
}

// Consumers: this warp is done with stage use k.
__device__ __forceinline__ void release_stage(StepShared& sh, uint32_t k) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&sh.empty[k % kStages]);
}

__device__ void step_producer(const Tile* __restrict__ tiles, int64_t n_tiles, int64_t bucket, int64_t n_blocks,
                              const float* master, const uint16_t* grad, const int8_t* mq, const uint8_t* vq,
                              const float2* scales, unsigned char* stages, StepShared& sh, int32_t* status) {
    uint32_t k = 0;
    bool timed_out = false;
    const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
    for (int64_t ti = blockIdx.x; ti < n_tiles && !timed_out; ti += gridDim.x) {
        const Tile t = tiles[ti];
        if (!tile_ok(t, bucket, n_blocks) || t.kind == TILE_ZERO) continue;
        const int64_t a0 = t.e0 & ~int64_t(kAlign - 1);
        const int64_t hi = t.e0 + t.n;
        const bool strip = t.kind == TILE_STRIP;
        const int passes = t.kind == TILE_WHOLE ? 1 : 2;
        const int64_t nch = t.kind == TILE_WHOLE ? 1 : strip ? strip_chunks(t) : large_chunks(t);
        for (int pass = 0; pass < passes && !timed_out; ++pass) {
            for (int64_t ch = 0; ch < nch; ++ch) {
                const uint32_t s = k % kStages;
                if (k >= kStages && !mbar_wait_bounded(&sh.empty[s], ((k / kStages) - 1u) & 1u)) {
                    timed_out = true;
                    break;
                }
                unsigned char* st = stages + s * kStageBytes;
                int64_t w0 = a0 + ch * kTile;
                uint32_t n16 = (uint32_t)((min(hi - w0, (int64_t)kTile) + 15) & ~int64_t(15));
                if (strip) {
                    int len;
                    strip_chunk(t, (int)ch, w0, len);
                    n16 = (uint32_t)len;
                }
                uint32_t bytes = n16 * (pass == 0 ? 8u : 4u);
                int64_t f = 0;
                uint32_t ns = 0;
                if (t.kind == TILE_WHOLE) {
                    f = t.blk0 & ~int64_t(1);
                    ns = (uint32_t)((t.blk0 + t.nblk - f + 1) & ~int64_t(1));
                    bytes += ns * 8u;
                }
                mbar_arrive_expect_tx(&sh.full[s], bytes);
                if (passes == 1) {
                    bulk_g2s(st + kOffG, grad + w0, n16 * 2u, &sh.full[s]);
                    bulk_g2s(st + kOffP, master + w0, n16 * 4u, &sh.full[s]);
                    bulk_g2s(st + kOffMQ, mq + w0, n16, &sh.full[s]);
                    bulk_g2s(st + kOffVQ, vq + w0, n16, &sh.full[s]);
                } else {
                    // Two-pass entries read grad and codes again in pass 2:
                    // ask L2 to keep them until then, and to drop them after.
                    const uint64_t pol = pass == 0 ? keep : drop;
                    bulk_g2s_hint(st + kOffG, grad + w0, n16 * 2u, &sh.full[s], pol);
                    if (pass == 0) bulk_g2s_hint(st + kOffP, master + w0, n16 * 4u, &sh.full[s], drop);
                    bulk_g2s_hint(st + kOffMQ, mq + w0, n16, &sh.full[s], pol);
                    bulk_g2s_hint(st + kOffVQ, vq + w0, n16, &sh.full[s], pol);
                }
                if (ns) bulk_g2s(st + kOffS, scales + f, ns * 8u, &sh.full[s]);
                ++k;
            }
        }
    }
    if (timed_out) {
        set_status(status, 1);
        // Let the copies already issued land before the CTA can go away.
        for (uint32_t j = k > (uint32_t)kStages ? k - kStages : 0u; j < k; ++j)
            mbar_wait_bounded(&sh.full[j % kStages], (j / kStages) & 1u);
    }
}

// A tile that is one block (the common case: 1-row blocks up to 4096
// elements).  Every consumer computes the block's dequantisation and
// quantisation factors itself, so only the absmax needs a barrier.  The
// absmax words alternate between two slots by tile parity: the slot of the
// next single-block tile is cleared here, after every reader of its last use
// has passed this tile's first barrier.
__device__ void single_tile(const Tile t, unsigned char* st, StepShared& sh, uint32_t par, float* master,
                            uint16_t* param, int8_t* mq, uint8_t* vq, float2* scales, const StepC2& c2,
                            float2 gs) {
    const int tid = threadIdx.x;
    const float2 sc = reinterpret_cast<const float2*>(st + kOffS)[t.blk0 & 1];
    const float2 dq = dequant_steps(sc);
    const float dqm = dq.x, dqv = dq.y;
    if (tid == 0) {
        sh.am1[par ^ 1u] = 0u;
        sh.ar1[par ^ 1u] = 0u;
    }
    const int64_t a0 = t.e0 & ~int64_t(kAlign - 1);
    const Out o{master + a0, param + a0, mq + a0, vq + a0};
    const int lo = (int)(t.e0 - a0), hi = lo + (int)t.n;
    float am = 0.f, ar = 0.f;
#pragma unroll
    for (int j = 0; j < kSub; ++j) {
        const int li = j * (kConsumers * kV) + kV * tid;
        if (!(li < hi && li + kV > lo)) continue;
        float m[kV], r[kV], vm, vr;
        if (li >= lo && li + kV <= hi)
            update8<true>(st, li, lo, hi, dqm, dqv, c2, gs, o, m, r, vm, vr);
        else
            update8<false>(st, li, lo, hi, dqm, dqv, c2, gs, o, m, r, vm, vr);
        am = fmaxf(am, vm);
        ar = fmaxf(ar, vr);
        stash_mr(st, li, m, r);
    }
    warp_max2(am, ar);
    if ((tid & 31) == 0) {
        atomicMax(&sh.am1[par], __float_as_uint(am));
        atomicMax(&sh.ar1[par], __float_as_uint(ar));
    }
    named_sync(kBarCons, kConsumers);
    const float AMm = __uint_as_float(sh.am1[par]), AMr = __uint_as_float(sh.ar1[par]);
    float qm[kV], qv[kV];
    {
        const float2 qf = quant_factors(make_float2(AMm, AMr));
        const float q1 = qf.x, q2 = qf.y;
#pragma unroll
        for (int i = 0; i < kV; ++i) {
            qm[i] = q1;
            qv[i] = q2;
        }
    }
    if (tid == 0) scales[t.blk0] = make_float2(AMm, AMr);
#pragma unroll
    for (int j = 0; j < kSub; ++j) {
        const int li = j * (kConsumers * kV) + kV * tid;
        if (!(li < hi && li + kV > lo)) continue;
        float m[kV], r[kV];
        unstash_mr(st, li, m, r);
        if (li >= lo && li + kV <= hi)
            store_codes8<true>(m, r, qm, qv, li, lo, hi, o);
        else
            store_codes8<false>(m, r, qm, qv, li, lo, hi, o);
    }
}

// Kinds of multi-block tiles, fixed per tile.
enum : int { W_MULTI8 = 1, W_MIXED = 2 };

// Several whole blocks: phase 1 updates the weights and parks m, sqrt(v) in
// the stage; block maxima meet in shared memory; phase 2 writes the codes.
//   W_MULTI8: blocks of a multiple of 8 elements, so each vector lies in one
//   block, found as umulhi(x, magic) = x / b.
//   W_MIXED: blocks not a multiple of 8 elements, per-element block numbers (rare).
template <int MODE>
__device__ void whole_tile(const Tile t, unsigned char* st, StepShared& sh, float* master, uint16_t* param,
                           int8_t* mq, uint8_t* vq, float2* scales, const StepC2& c2, float2 gs) {
    const int tid = threadIdx.x;
    const int nb = t.nblk;
    if (tid < nb) {
        const float2 sc = reinterpret_cast<const float2*>(st + kOffS)[(t.blk0 & 1) + tid];
        const float2 dq = dequant_steps(sc);
        sh.dqm[tid] = dq.x;
        sh.dqv[tid] = dq.y;
        sh.am[tid] = 0u;
        sh.ar[tid] = 0u;
    }
    named_sync(kBarCons, kConsumers);

    const int64_t a0 = t.e0 & ~int64_t(kAlign - 1);
    const Out o{master + a0, param + a0, mq + a0, vq + a0};
    const int lo = (int)(t.e0 - a0), hi = lo + (int)t.n;  // local range of the tile's elements
    const uint32_t b = (uint32_t)t.b, magic = t.magic;
#pragma unroll
    for (int j = 0; j < kSub; ++j) {
        const int li = j * (kConsumers * kV) + kV * tid;
        const bool any = li < hi && li + kV > lo;
        const bool full = li >= lo && li + kV <= hi;
        float m[kV], r[kV];
        if (MODE == W_MULTI8) {
            int key = -1;
            float am = 0.f, ar = 0.f;
            if (any) {
                key = (int)__umulhi((uint32_t)(max(li, lo) - lo), magic);
                if (full)
                    update8<true>(st, li, lo, hi, sh.dqm[key], sh.dqv[key], c2, gs, o, m, r, am, ar);
                else
                    update8<false>(st, li, lo, hi, sh.dqm[key], sh.dqv[key], c2, gs, o, m, r, am, ar);
                stash_mr(st, li, m, r);
            }
            block_max_to_smem(key, am, ar, sh);
        } else {
            if (any) {
                const StepC c{c2.b1.x, c2.omb1.x, c2.b2.x, c2.omb2.x, c2.eps_hat.x, c2.step_hat.x, c2.decay.x, gs.x};
                In8 x;
                load8<false>(x, st, li, lo, hi, true);
#pragma unroll
                for (int i = 0; i < kV; ++i) {
                    const int e = li + i;
                    const int blk = (e >= lo && e < hi) ? (int)((uint32_t)(e - lo) / b) : 0;
                    new_m_r(g_of(x, i), sbyte_to_f(x.mq[i >> 2], i & 3), ubyte_to_f(x.vq[i >> 2], i & 3), sh.dqm[blk], sh.dqv[blk], c, m[i],
                            r[i]);
                    x.p[i] = new_p(x.p[i], m[i], r[i], c);
                    if (e >= lo && e < hi) {
                        atomicMax(&sh.am[blk], __float_as_uint(fabsf(m[i])));
                        atomicMax(&sh.ar[blk], __float_as_uint(r[i]));
                    }
                }
                store_p8<false>(x.p, li, lo, hi, o);
                stash_mr(st, li, m, r);
            }
        }
    }
    named_sync(kBarCons, kConsumers);
    if (tid < nb) {
        const float AMm = __uint_as_float(sh.am[tid]), AMr = __uint_as_float(sh.ar[tid]);
        const float2 qf = quant_factors(make_float2(AMm, AMr));
        sh.qm[tid] = qf.x;
        sh.qv[tid] = qf.y;
        scales[t.blk0 + tid] = make_float2(AMm, AMr);
    }
    named_sync(kBarCons, kConsumers);
#pragma unroll
    for (int j = 0; j < kSub; ++j) {
        const int li = j * (kConsumers * kV) + kV * tid;
        if (!(li < hi && li + kV > lo)) continue;
        const bool full = li >= lo && li + kV <= hi;
        float m[kV], r[kV], qm[kV], qv[kV];
        unstash_mr(st, li, m, r);
        if (MODE == W_MIXED) {
#pragma unroll
            for (int i = 0; i < kV; ++i) {
                const int e = li + i;
                const int blk = (e >= lo && e < hi) ? (int)((uint32_t)(e - lo) / b) : 0;
                qm[i] = sh.qm[blk];
                qv[i] = sh.qv[blk];
            }
        } else {
            const int key = (int)__umulhi((uint32_t)(max(li, lo) - lo), magic);
            const float q1 = sh.qm[key], q2 = sh.qv[key];
#pragma unroll
            for (int i = 0; i < kV; ++i) {
                qm[i] = q1;
                qv[i] = q2;
            }
        }
        if (full)
            store_codes8<true>(m, r, qm, qv, li, lo, hi, o);
        else
            store_codes8<false>(m, r, qm, qv, li, lo, hi, o);
    }
}

// A block longer than a tile: pass 1 over its chunks updates the weights and
// finds the absmax; pass 2 reloads grad and old codes, recomputes m and
// sqrt(v) and writes the codes.
__device__ int64_t large_tile(const Tile t, uint32_t k, unsigned char* stages, StepShared& sh, float* master,
                           uint16_t* param, int8_t* mq, uint8_t* vq, float2* scales, const StepC2& c2,
                           float2 gs, int32_t* status) {
    const int tid = threadIdx.x;
    const float2 sc = scales[t.blk0];
    const float2 dq = dequant_steps(sc);
    const float dqm = dq.x, dqv = dq.y;
    const int64_t a0 = t.e0 & ~int64_t(kAlign - 1);
    const int64_t nch = large_chunks(t);

    float am = 0.f, ar = 0.f;
    for (int64_t ch = 0; ch < nch; ++ch) {
        if (!wait_stage(sh, k, status)) return -1;
        const unsigned char* st = stages + (k % kStages) * kStageBytes;
        const int64_t w0 = a0 + ch * kTile;
        const Out o{master + w0, param + w0, mq + w0, vq + w0};
        const int lo = (int)max(t.e0 - w0, (int64_t)0), hi = (int)min(t.e0 + t.n - w0, (int64_t)kTile);
#pragma unroll
        for (int j = 0; j < kSub; ++j) {
            const int li = j * (kConsumers * kV) + kV * tid;
            if (!(li < hi && li + kV > lo)) continue;
            float m[kV], r[kV], vm, vr;
            if (li >= lo && li + kV <= hi)
                update8<true>(st, li, lo, hi, dqm, dqv, c2, gs, o, m, r, vm, vr);
            else
                update8<false>(st, li, lo, hi, dqm, dqv, c2, gs, o, m, r, vm, vr);
            am = fmaxf(am, vm);
            ar = fmaxf(ar, vr);
        }
        release_stage(sh, k);
        ++k;
    }
    warp_max2(am, ar);
    if ((tid & 31) == 0) {
        sh.red[0][tid >> 5] = am;
        sh.red[1][tid >> 5] = ar;
    }
    named_sync(kBarCons, kConsumers);
    if (tid == 0) {
        float a = 0.f, q = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            a = fmaxf(a, sh.red[0][w]);
            q = fmaxf(q, sh.red[1][w]);
        }
        const float2 qf = quant_factors(make_float2(a, q));
        sh.qm[0] = qf.x;
        sh.qv[0] = qf.y;
        scales[t.blk0] = make_float2(a, q);
    }
    named_sync(kBarCons, kConsumers);
    const float qm1 = sh.qm[0], qv1 = sh.qv[0];
    float qm[kV], qv[kV];
#pragma unroll
    for (int i = 0; i < kV; ++i) {
        qm[i] = qm1;
        qv[i] = qv1;
    }
    for (int64_t ch = 0; ch < nch; ++ch) {
        if (!wait_stage(sh, k, status)) return -1;
        const unsigned char* st = stages + (k % kStages) * kStageBytes;
        const int64_t w0 = a0 + ch * kTile;
        const Out o{master + w0, param + w0, mq + w0, vq + w0};
        const int lo = (int)max(t.e0 - w0, (int64_t)0), hi = (int)min(t.e0 + t.n - w0, (int64_t)kTile);
#pragma unroll
        for (int j = 0; j < kSub; ++j) {
            const int li = j * (kConsumers * kV) + kV * tid;
            if (!(li < hi && li + kV > lo)) continue;
            const bool full = li >= lo && li + kV <= hi;
            In8 x;
            float m[kV], r[kV];
            if (full)
                load8<true>(x, st, li, lo, hi, false);
            else
                load8<false>(x, st, li, lo, hi, false);
            mr8(x, dqm, dqv, c2, gs, m, r);
            if (full)
                store_codes8<true>(m, r, qm, qv, li, lo, hi, o);
            else
                store_codes8<false>(m, r, qm, qv, li, lo, hi, o);
        }
        release_stage(sh, k);
        ++k;
    }
    return k;
}

// A STRIP entry (2-D blocks): the columns of a chunk that a thread's vector
// covers are the same in every chunk (whole rows per chunk, every row start
// 16-element aligned), so each thread keeps its vectors' tile index, old
// dequantisation steps and running maxima in registers across the chunks.
// Pass 1 updates the weights; the tiles' maxima meet in shared memory;
// pass 2 reloads grad and old codes, recomputes m and sqrt(v) and writes the
// codes.  Vectors never straddle tiles (tile width and cols are multiples
// of 16).
__device__ int64_t strip_tile(const Tile t, uint32_t k, unsigned char* stages, StepShared& sh, float* master,
                           uint16_t* param, int8_t* mq, uint8_t* vq, float2* scales, const StepC2& c2,
                           float2 gs, int32_t* status) {
    const int tid = threadIdx.x;
    const int C = t.b, W = (int)t.magic;
    const int G = ((int)t.n + W - 1) / W;
    const int nch = strip_chunks(t);
    const int full = C <= kTile ? strip_rows_per_chunk(t) * C : (int)t.n;  // elements of a full chunk
    int gi[kSub];
    float2 dq[kSub];
    float am[kSub], ar[kSub];
#pragma unroll
    for (int j = 0; j < kSub; ++j) {
        const int x = j * (kConsumers * kV) + kV * tid;
        gi[j] = x < full ? (C <= kTile ? x % C : x) / W : -1;
        dq[j] = gi[j] >= 0 ? dequant_steps(scales[t.blk0 + gi[j]]) : make_float2(0.f, 0.f);
        am[j] = 0.f;
        ar[j] = 0.f;
    }
    if (tid < G) {
        sh.am[tid] = 0u;
        sh.ar[tid] = 0u;
    }
    for (int ch = 0; ch < nch; ++ch) {
        if (!wait_stage(sh, k, status)) return -1;
        const unsigned char* st = stages + (k % kStages) * kStageBytes;
        int64_t w0;
        int len;
        strip_chunk(t, ch, w0, len);
        const Out o{master + w0, param + w0, mq + w0, vq + w0};
#pragma unroll
        for (int j = 0; j < kSub; ++j) {
            const int li = j * (kConsumers * kV) + kV * tid;
            if (li >= len) continue;
            float m[kV], r[kV], vm, vr;
            update8<true>(st, li, 0, len, dq[j].x, dq[j].y, c2, gs, o, m, r, vm, vr);
            am[j] = fmaxf(am[j], vm);
            ar[j] = fmaxf(ar[j], vr);
        }
        release_stage(sh, k);
        ++k;
    }
#pragma unroll
    for (int j = 0; j < kSub; ++j) block_max_to_smem(gi[j], am[j], ar[j], sh);
    named_sync(kBarCons, kConsumers);
    if (tid < G) {
        const float AMm = __uint_as_float(sh.am[tid]), AMr = __uint_as_float(sh.ar[tid]);
        const float2 qf = quant_factors(make_float2(AMm, AMr));
        sh.qm[tid] = qf.x;
        sh.qv[tid] = qf.y;
        scales[t.blk0 + tid] = make_float2(AMm, AMr);
    }
    named_sync(kBarCons, kConsumers);
    float q1[kSub], q2[kSub];
#pragma unroll
    for (int j = 0; j < kSub; ++j) {
        q1[j] = gi[j] >= 0 ? sh.qm[gi[j]] : 0.f;
        q2[j] = gi[j] >= 0 ? sh.qv[gi[j]] : 0.f;
    }
    for (int ch = 0; ch < nch; ++ch) {
        if (!wait_stage(sh, k, status)) return -1;
        const unsigned char* st = stages + (k % kStages) * kStageBytes;
        int64_t w0;
        int len;
        strip_chunk(t, ch, w0, len);
        const Out o{master + w0, param + w0, mq + w0, vq + w0};
#pragma unroll
        for (int j = 0; j < kSub; ++j) {
            const int li = j * (kConsumers * kV) + kV * tid;
            if (li >= len) continue;
            In8 x;
            float m[kV], r[kV], qm[kV], qv[kV];
            load8<true>(x, st, li, 0, len, false);
            mr8(x, dq[j].x, dq[j].y, c2, gs, m, r);
#pragma unroll
            for (int i = 0; i < kV; ++i) {
                qm[i] = q1[j];
                qv[i] = q2[j];
            }
            store_codes8<true>(m, r, qm, qv, li, 0, len, o);
        }
        release_stage(sh, k);
        ++k;
    }
    return k;
}

__device__ void zero_tile(const Tile t, uint16_t* param) {
    const int64_t lo = t.e0, hi = t.e0 + t.n;
    const int64_t a0 = t.e0 & ~int64_t(kAlign - 1);
    for (int64_t vb = a0 + 8 * (int64_t)threadIdx.x; vb < hi; vb += 8 * (int64_t)kConsumers) {
        if (vb >= lo && vb + 8 <= hi) {
            __stcs(reinterpret_cast<uint4*>(param + vb), make_uint4(0, 0, 0, 0));
        } else {
            for (int i = 0; i < 8; ++i)
                if (vb + i >= lo && vb + i < hi) param[vb + i] = 0;
        }
    }
}

__global__ void __launch_bounds__(kStepThreads, DBUF_STEP_MIN_CTAS)
    adam8_step_kernel(const Tile* __restrict__ tiles, int64_t n_tiles, int64_t bucket, float* master,
                      uint16_t* param, const uint16_t* grad, int8_t* mq, uint8_t* vq, float2* scales,
                      int64_t n_blocks, const __grid_constant__ StepC2 cp, const float* gscale_dev,
                      int32_t* status) {
    extern __shared__ __align__(128) unsigned char stages[];
    __shared__ StepShared sh;
    const int tid = threadIdx.x;
    // The step constants stay in the parameter space (paired operands read
    // from the constant bank, no registers held).  grad_scale comes from
    // device memory when a preceding kernel chose it (global-norm clipping),
    // so no host round trip is needed.
    const float2 gs = gscale_dev ? dup(*gscale_dev) : cp.gscale;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], kConsumerWarps);
        }
        fence_barrier_init();
        sh.am1[0] = sh.am1[1] = sh.ar1[0] = sh.ar1[1] = 0u;
    }
    __syncthreads();
    if (tid >= kConsumers) {  // producer warp: one lane issues all copies
        if (tid == kConsumers)
            step_producer(tiles, n_tiles, bucket, n_blocks, master, grad, mq, vq, scales, stages, sh, status);
        return;
    }
    uint32_t k = 0, nsingle = 0;
    for (int64_t ti = blockIdx.x; ti < n_tiles; ti += gridDim.x) {
        const Tile t = tiles[ti];
        if (!tile_ok(t, bucket, n_blocks)) {
            if (tid == 0) set_status(status, 2);
            continue;
        }
        if (t.kind == TILE_ZERO) {
            zero_tile(t, param);
        } else if (t.kind == TILE_WHOLE) {
            if (!wait_stage(sh, k, status)) return;
            unsigned char* st = stages + (k % kStages) * kStageBytes;
            if (t.nblk == 1) {
                single_tile(t, st, sh, nsingle & 1u, master, param, mq, vq, scales, cp, gs);
                ++nsingle;
            } else if ((t.b & 7) == 0)
                whole_tile<W_MULTI8>(t, st, sh, master, param, mq, vq, scales, cp, gs);
            else
                whole_tile<W_MIXED>(t, st, sh, master, param, mq, vq, scales, cp, gs);
            release_stage(sh, k);
            ++k;
        } else {
            const int64_t nk = t.kind == TILE_STRIP
                                   ? strip_tile(t, k, stages, sh, master, param, mq, vq, scales, cp, gs, status)
                                   : large_tile(t, k, stages, sh, master, param, mq, vq, scales, cp, gs, status);
            if (nk < 0) return;
            k = (uint32_t)nk;
        }
    }
}

}  // namespace dbuf_k

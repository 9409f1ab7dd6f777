// Correctly rounded square root and division without the library calls'
// special-case branches, on argument ranges the callers test first.
//
// Square root, for v >= 2^-100 (the step's v = b2*v_old + (1-b2)*g^2 is far
// above that for any gradient larger than about 1e-15).  Method (Markstein,
// "IA-64 and Elementary Functions", 2000, ch. 8: one Newton correction of
// sqrt(v) with an exact residual): y ~ 1/sqrt(v) from the hardware
// approximation, s = v*y ~ sqrt(v), e = v - s*s exactly by one FMA,
// r = s + e*(y/2).  Checked exhaustively against __fsqrt_rn on the GPU
// (tests/test_gpu_fastmath.py): equal for every float in [2^-100, FLT_MAX];
// below about 2^-103 the residual underflows and it is not, so callers test
// the argument first (sqrt_fast_ok) and use __fsqrt_rn otherwise.
//
// Division a/d (same book, ch. 8, the quotient correction with a correctly
// rounded reciprocal): y0 ~ 1/d from the hardware approximation, one Newton
// step y = y0 + y0(1 - d*y0) (equal to 1/d rounded to nearest for every d
// in the range below, checked exhaustively), q0 = a*y, the residual a - d*q0
// is exact by one FMA, and q = q0 + residual*y is a/d correctly rounded
// (Markstein's theorem: y the rounded reciprocal, q0 within an ulp of a/d).
// The ranges keep every intermediate normal: d in [2^-60, 2^64],
// |a| in [2^-61, 2^68]; checked against __fdiv_rn on the GPU over random
// and structured pairs (tests/test_gpu_fastmath.py).
#pragma once

#include <cstdint>

namespace dbuf_k {

__device__ __forceinline__ float rsqrt_approx(float v) {
    float y;
    asm("rsqrt.approx.f32 %0, %1;" : "=f"(y) : "f"(v));
    return y;
}

__device__ __forceinline__ float rcp_approx(float d) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(d));
    return y;
}

__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Lower end of the exactly checked range: bit pattern of 2^-100.
constexpr uint32_t kSqrtFastMinBits = 0x0D800000u;

__device__ __forceinline__ bool sqrt_fast_ok(float v) { return __float_as_uint(v) >= kSqrtFastMinBits; }

// sqrt of two floats in [2^-100, FLT_MAX], correctly rounded.
__device__ __forceinline__ float2 sqrt2_fast(float2 v) {
    const float2 y = make_float2(rsqrt_approx(v.x), rsqrt_approx(v.y));
    const float2 s = mul2_rn(v, y);
    const float2 h = mul2_rn(y, make_float2(0.5f, 0.5f));
    const float2 e = fma2_rn(make_float2(-s.x, -s.y), s, v);
    return fma2_rn(e, h, s);
}

// Ranges of div2_fast (see the header comment).
constexpr float kDivMinD = 0x1p-60f, kDivMaxD = 0x1p64f;
constexpr float kDivMinA = 0x1p-61f, kDivMaxA = 0x1p68f;

// The reciprocal of two floats in [2^-60, 2^64], rounded to nearest.
__device__ __forceinline__ float2 rcp2_fast(float2 d) {
    const float2 y0 = make_float2(rcp_approx(d.x), rcp_approx(d.y));
    const float2 e = fma2_rn(make_float2(-d.x, -d.y), y0, make_float2(1.f, 1.f));
    return fma2_rn(y0, e, y0);
}

// a/d of two pairs, correctly rounded, for d and |a| in the ranges above.
__device__ __forceinline__ float2 div2_fast(float2 a, float2 d) {
    const float2 y = rcp2_fast(d);
    const float2 q0 = mul2_rn(a, y);
    const float2 r = fma2_rn(make_float2(-d.x, -d.y), q0, a);
    return fma2_rn(r, y, q0);
}

// Per-block factors of the 8-bit codes, pair (m, sqrt(v)) at once.
//   dequantisation steps (scale_m/127, scale_v/255): the quotient correction
//   with the constant reciprocals rounded to nearest, exact for every finite
//   nonzero scale (checked exhaustively); zeros are returned as they are,
//   infinite or NaN scales take IEEE division.
//   quantisation factors (127/max|m|, 255/max sqrt(v)): div2_fast's sequence
//   for maxima in [2^-60, 2^64] (checked exhaustively), IEEE division
//   otherwise, 0 for a zero maximum.
__device__ __forceinline__ float2 dequant_steps(float2 sc) {
    if (fabsf(sc.x) <= 3.402823466e38f && fabsf(sc.y) <= 3.402823466e38f) {
        const float2 c = make_float2(127.f, 255.f), cr = make_float2(1.f / 127.f, 1.f / 255.f);
        const float2 q0 = mul2_rn(sc, cr);
        const float2 r = fma2_rn(make_float2(-c.x, -c.y), q0, sc);
        const float2 q = fma2_rn(r, cr, q0);
        // a zero scale gives that zero, sign included (the correction would turn -0 into +0)
        return make_float2(sc.x == 0.f ? sc.x : q.x, sc.y == 0.f ? sc.y : q.y);
    }
    return make_float2(__fdiv_rn(sc.x, 127.f), __fdiv_rn(sc.y, 255.f));
}

__device__ __forceinline__ float2 quant_factors(float2 am) {
    float2 q;
    if (am.x >= kDivMinD && am.x <= kDivMaxD && am.y >= kDivMinD && am.y <= kDivMaxD)
        q = div2_fast(make_float2(127.f, 255.f), am);
    else
        q = make_float2(__fdiv_rn(127.f, am.x), __fdiv_rn(255.f, am.y));
    return make_float2(am.x > 0.f ? q.x : 0.f, am.y > 0.f ? q.y : 0.f);
}

}  // namespace dbuf_k

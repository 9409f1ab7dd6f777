// Correctly rounded square root without the library call's special-case
// branches, for arguments v >= 2^-100 (the step's v = b2*v_old + (1-b2)*g^2
// is far above that for any gradient larger than about 1e-15).
//
// Method (Markstein, "IA-64 and Elementary Functions", 2000, ch. 8: one
// Newton correction of sqrt(v) with an exact residual): y ~ 1/sqrt(v) from
// the hardware approximation, s = v*y ~ sqrt(v), e = v - s*s exactly by one
// FMA, r = s + e*(y/2).  Checked exhaustively against __fsqrt_rn on the GPU
// (tests/test_gpu_fastmath.py): equal for every float in [2^-100, FLT_MAX];
// below about 2^-103 the residual underflows and it is not, so callers test
// the argument first (sqrt_fast_ok) and use __fsqrt_rn otherwise.
#pragma once

#include <cstdint>

namespace dbuf_k {

__device__ __forceinline__ float rsqrt_approx(float v) {
    float y;
    asm("rsqrt.approx.f32 %0, %1;" : "=f"(y) : "f"(v));
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

}  // namespace dbuf_k

// NVFP4 block quantization shared by the append kernel and the fused
// projection epilogue (sm_100a device code).  Format and arithmetic as the
// append kernel's header states: s_g = fl32(amax / 2688) (1 if not a normal
// float), s_b = E4M3_RNE(min(fl32(amax16 / fl32(6 s_g)), 448)),
// q_i = E2M1_RNE_sat(fl32(x_i / fl32(s_b s_g))), no negative zero; the
// shared-divisor quotients by Markstein's correctly rounded division inside
// 2^-64 <= d <= 2^64, IEEE division outside.
#pragma once

#include <cstdint>

namespace nvkv {
namespace q4 {

// max |x| over the eight bf16 values of two words pairs, as a float.
__device__ __forceinline__ uint32_t absmax_bits(uint4 a)
{
    uint32_t m = __vmaxu2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, __vmaxu2(a.z & 0x7FFF7FFFu, a.w & 0x7FFF7FFFu));
    return m;
}

__device__ __forceinline__ float halves_max(uint32_t m)
{
    const uint32_t hi = m >> 16, lo = m & 0xFFFFu;
    return __uint_as_float((hi > lo ? hi : lo) << 16);
}

__device__ __forceinline__ float global_scale_from_amax(uint32_t amax_bits)
{
    float s = __fdiv_rn(__uint_as_float(amax_bits), 2688.0f);
    return (s >= 1.17549435e-38f) ? s : 1.0f;
}

// E4M3 code of t >= 0, round-to-nearest-even, saturating at 448 (hardware cvt).
__device__ __forceinline__ uint32_t e4m3_code(float t)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
    return r & 0xFFu;
}

// Value of a non-negative finite E4M3 code (exact).
__device__ __forceinline__ float e4m3_value(uint32_t c)
{
    const uint32_t e = c >> 3, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
}

// Eight E2M1 codes, element i in nibble i (hardware cvt: the second source
// operand lands in the low nibble).
__device__ __forceinline__ uint32_t e2m1x8(const float *y)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]),
          "f"(y[7]));
    return r;
}

// Clear the sign of every nibble whose magnitude is zero (no negative zero).
__device__ __forceinline__ uint32_t drop_negative_zero(uint32_t w)
{
    const uint32_t mag = w & 0x77777777u;
    const uint32_t nonzero = (mag + 0x77777777u) & 0x88888888u;
    return mag | (w & nonzero);
}

__device__ __forceinline__ void unpack_bf16x8(uint4 a, float *x)
{
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Codes of one 16-element block (bf16 in w0, w1) with global scale sg:
// returns the E4M3 scale code, writes the 16 codes (element i in nibble i of
// c.x | c.y << 32).
// The same block rule for 16 float inputs (rotated keys), with IEEE division
// for every quotient (the shared-divisor shortcut is only verified on bf16
// inputs).
__device__ __forceinline__ uint32_t quantize_block_f32(const float *x, float sg, uint2 &c)
{
    float amax16 = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax16 = fmaxf(amax16, fabsf(x[i]));
    const float ratio = __fdiv_rn(amax16, __fmul_rn(6.0f, sg));
    const uint32_t sb_code = e4m3_code(ratio);
    const float sb = e4m3_value(sb_code);
    c = make_uint2(0u, 0u);
    if (sb == 0.0f) return sb_code;
    const float d = __fmul_rn(sb, sg);
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fdiv_rn(x[i], d);
    c.x = drop_negative_zero(e2m1x8(y));
    c.y = drop_negative_zero(e2m1x8(y + 8));
    return sb_code;
}

__device__ __forceinline__ uint32_t quantize_block(uint4 w0, uint4 w1, float sg, uint2 &c)
{
    const float amax16 = halves_max(__vmaxu2(absmax_bits(w0), absmax_bits(w1)));
    const float ratio = __fdiv_rn(amax16, __fmul_rn(6.0f, sg));
    const uint32_t sb_code = e4m3_code(ratio);
    const float sb = e4m3_value(sb_code);
    c = make_uint2(0u, 0u);
    if (sb == 0.0f) return sb_code;
    const float d = __fmul_rn(sb, sg);
    float x[16], y[16];
    unpack_bf16x8(w0, x);
    unpack_bf16x8(w1, x + 8);
    const float r = __frcp_rn(d);
    if (d >= 0x1p-64f && d <= 0x1p64f && amax16 * r < 0x1p64f) {
        // y = RN(q + (x - q d) r) with q = RN(x r), two elements per operation
        const float2 r2 = make_float2(r, r), nd2 = make_float2(-d, -d);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float2 xx = make_float2(x[i], x[i + 1]);
            const float2 q = __fmul2_rn(xx, r2);
            const float2 yy = __ffma2_rn(__ffma2_rn(q, nd2, xx), r2, q);
            y[i] = yy.x;
            y[i + 1] = yy.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = __fdiv_rn(x[i], d);
    }
    c.x = drop_negative_zero(e2m1x8(y));
    c.y = drop_negative_zero(e2m1x8(y + 8));
    return sb_code;
}

}  // namespace q4
}  // namespace nvkv

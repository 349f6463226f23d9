// NVFP4 arithmetic on the GPU: the per-group quantization rule in fp32 IEEE operations
// with explicit rounding intrinsics (no multiply-add is contracted; codes and scales
// must match the CPU oracle bit for bit) and the hardware E2M1 and E4M3 conversions.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace mq {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// E4M3 (fn) encode of a non-negative finite fp32: round to nearest even, saturate to 448
// (0x7E). cvt.rn.satfinite.e4m3x2.f32 implements exactly this rule: it was compared on
// B200 with an encoder written from the format's bit layout (normal grid 2^(E-7) * 1.m,
// subnormal grid m * 2^-9, ties to the even code) over every non-negative finite fp32
// value, with no difference. The second source operand lands in the low byte.
__device__ __forceinline__ uint32_t e4m3_encode_nonneg(float s) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(s));
    return h & 0xFFu;
}

// Value of a non-negative E4M3 byte (0x00..0x7E).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e == 0 ? __fmul_rn((float)m, 0.001953125f) : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Maximum of three fp32 values (sm_100 three-input max; exact).
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Packed fp32 multiply (sm_100 mul.rn.f32x2): each lane is one IEEE fp32 multiply with
// round-to-nearest-even, bit-identical to __fmul_rn (a product's sign, zeros included,
// is the xor of the operands' signs). Packed add/sub/fma are not used: on B200,
// sub.rn.f32x2 returned -0 for (-x) - (-x), where IEEE round-to-nearest gives +0 (the sign
// of a zero residual is part of its code), and Delta values computed with it for e' =
// R - deqR (only ever squared) differed from the IEEE scalar path.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Eight scaled values -> eight E2M1 codes packed in a word (element 0 in the low nibble
// of byte 0). The E2M1 rule: round to nearest with ties to the even code, saturate at 6,
// keep the sign (-0.1 -> 0x8). cvt.rn.satfinite.e2m1x2 implements exactly this rule:
// it was compared on B200 with an encoder written from the format's bit layout over
// every finite fp32 value, with no difference.
__device__ __forceinline__ uint32_t e2m1x8(float q0, float q1, float q2, float q3, float q4, float q5, float q6,
                                           float q7) {
    uint32_t w;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(w)
        : "f"(q0), "f"(q1), "f"(q2), "f"(q3), "f"(q4), "f"(q5), "f"(q6), "f"(q7));
    return w;
}

// Signed E2M1 values of the eight codes of a word (exact in f16, widened to fp32).
__device__ __forceinline__ void e2m1x8_values(uint32_t w, float* v) {
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __half2 x = *reinterpret_cast<const __half2*>(&h[j]);
        const float2 f = __half22float2(x);
        v[2 * j] = f.x;
        v[2 * j + 1] = f.y;
    }
}

// Codes of 16 values that all round to a signed zero (the group scale is zero).
__device__ __forceinline__ uint32_t sign_nibbles8(const float* a) {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) w |= ((__float_as_uint(a[i]) >> 28) & 8u) << (4 * i);
    return w;
}

// One 16-element group with tensor scale g (g6 = fp32(6 g)):
//   s = amax / g6; sf = E4M3(s); d = dec(sf) * g; r = 1 / d;
//   code_i = E2M1(a_i * r) (a signed zero if d == 0); deq_i = val(code_i) * d.
// Returns the scale byte; codes (element 2j in the low nibble of byte j) in lo/hi.
__device__ __forceinline__ uint32_t nvfp4_group(const float (&a)[16], float g, float g6, uint32_t& lo, uint32_t& hi,
                                                float (&deq)[16]) {
    float amax = max3(fabsf(a[0]), fabsf(a[1]), fabsf(a[2]));
#pragma unroll
    for (int i = 3; i < 15; i += 2) amax = max3(amax, fabsf(a[i]), fabsf(a[i + 1]));
    amax = fmaxf(amax, fabsf(a[15]));
    const float s = __fdiv_rn(amax, g6);
    const uint32_t sf = e4m3_encode_nonneg(s);
    const float d = __fmul_rn(e4m3_value(sf), g);
    if (d > 0.0f) {
        const float r = __frcp_rn(d);
        const float2 rr = make_float2(r, r);
        float2 q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = mul2(make_float2(a[2 * j], a[2 * j + 1]), rr);
        lo = e2m1x8(q[0].x, q[0].y, q[1].x, q[1].y, q[2].x, q[2].y, q[3].x, q[3].y);
        hi = e2m1x8(q[4].x, q[4].y, q[5].x, q[5].y, q[6].x, q[6].y, q[7].x, q[7].y);
    } else {
        lo = sign_nibbles8(a);
        hi = sign_nibbles8(a + 8);
    }
    float v[16];
    e2m1x8_values(lo, v);
    e2m1x8_values(hi, v + 8);
    const float2 dd = make_float2(d, d);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 t = mul2(make_float2(v[2 * j], v[2 * j + 1]), dd);
        deq[2 * j] = t.x;
        deq[2 * j + 1] = t.y;
    }
    return sf;
}

// The dequantization step d = fp32(dec(sf) * g) and its reciprocal r = fp32(1 / d) (0 when
// d = 0) of every E4M3 scale code 0..127 for tensor scale g, as (d, r) pairs: the same
// operations nvfp4_group performs per group, done once per CTA. The CTA's threads fill it
// (the caller synchronizes before use).
__device__ __forceinline__ void nvfp4_scale_table(float g, float2* tab) {
    for (int c = threadIdx.x; c < 128; c += blockDim.x) {
        const float d = __fmul_rn(e4m3_value((uint32_t)c), g);
        tab[c] = make_float2(d, d > 0.0f ? __frcp_rn(d) : 0.0f);
    }
}

// nvfp4_group with d and r looked up in a table from nvfp4_scale_table (bit-identical).
__device__ __forceinline__ uint32_t nvfp4_group_tab(const float (&a)[16], float g6, const float2* tab, uint32_t& lo,
                                                    uint32_t& hi, float (&deq)[16]) {
    float amax = max3(fabsf(a[0]), fabsf(a[1]), fabsf(a[2]));
#pragma unroll
    for (int i = 3; i < 15; i += 2) amax = max3(amax, fabsf(a[i]), fabsf(a[i + 1]));
    amax = fmaxf(amax, fabsf(a[15]));
    const uint32_t sf = e4m3_encode_nonneg(__fdiv_rn(amax, g6));
    const float2 dr = tab[sf];
    const float d = dr.x;
    if (d > 0.0f) {
        const float2 rr = make_float2(dr.y, dr.y);
        float2 q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = mul2(make_float2(a[2 * j], a[2 * j + 1]), rr);
        lo = e2m1x8(q[0].x, q[0].y, q[1].x, q[1].y, q[2].x, q[2].y, q[3].x, q[3].y);
        hi = e2m1x8(q[4].x, q[4].y, q[5].x, q[5].y, q[6].x, q[6].y, q[7].x, q[7].y);
    } else {
        lo = sign_nibbles8(a);
        hi = sign_nibbles8(a + 8);
    }
    float v[16];
    e2m1x8_values(lo, v);
    e2m1x8_values(hi, v + 8);
    const float2 dd = make_float2(d, d);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 t = mul2(make_float2(v[2 * j], v[2 * j + 1]), dd);
        deq[2 * j] = t.x;
        deq[2 * j + 1] = t.y;
    }
    return sf;
}

// Byte offset of (row r, group q) in the GEMM's tiled scale layout of a matrix with
// `cols` columns: 512-byte chunks per (128-row tile, 4 groups), (t%32)*16 + (t/32)*4 + q%4.
__device__ __forceinline__ int64_t sf_swz_offset(int64_t r, int64_t q, int cols) {
    const int64_t ks = cols / 64, t = r & 127;
    return (((r >> 7) * ks + (q >> 2)) << 9) + ((t & 31) << 4) + ((t >> 5) << 2) + (q & 3);
}

}  // namespace mq

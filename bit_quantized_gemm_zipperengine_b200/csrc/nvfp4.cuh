// NVFP4 arithmetic on the GPU: E2M1 / E4M3 encoders written from the bit layouts and
// the per-group quantization rule, in fp32 IEEE operations with explicit rounding
// intrinsics so that no multiply-add is contracted (codes and scales must match the
// CPU oracle bit for bit).
#pragma once

#include <cstdint>

namespace mq {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// E2M1 code of v: round to nearest, ties to the even code, saturate at 6, keep the sign.
// The magnitude code counts the grid midpoints below |v|; a midpoint itself goes to
// the even neighbour, hence the alternating strict / non-strict comparisons.
__device__ __forceinline__ uint32_t e2m1_encode(float v) {
    const float a = fabsf(v);
    uint32_t m = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
    return m | ((__float_as_uint(v) >> 28) & 8u);
}

// |value| of an E2M1 magnitude code (0..7): {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
__device__ __forceinline__ float e2m1_mag(uint32_t m) {
    // exponent field e = m >> 1 (bias 1), mantissa bit m & 1; e = 0 is subnormal (m * 0.5)
    const uint32_t e = m >> 1, f = m & 1u;
    return e == 0 ? 0.5f * (float)f : __uint_as_float(((e + 126u) << 23) | (f << 22));
}

// E4M3 (fn) encode of a non-negative finite fp32: round to nearest even, saturate to 448.
__device__ __forceinline__ uint32_t e4m3_encode_nonneg(float s) {
    if (s >= 448.0f) return 0x7Eu;
    if (s < 0.015625f) {  // below 2^-6 the grid is m * 2^-9 (m = 8 is 2^-6, code 0x08)
        return (uint32_t)__float2int_rn(__fmul_rn(s, 512.0f));
    }
    const uint32_t u = __float_as_uint(s);
    int E = (int)((u >> 23) & 0xFFu) - 127;  // -6 .. 8
    uint32_t keep = (u >> 20) & 7u;
    const uint32_t rest = u & 0xFFFFFu, half = 0x80000u;
    if (rest > half || (rest == half && (keep & 1u))) ++keep;
    if (keep == 8u) { keep = 0; ++E; }
    if (E > 8 || (E == 8 && keep > 6u)) return 0x7Eu;
    return ((uint32_t)(E + 7) << 3) | keep;
}

// Value of a non-negative E4M3 byte (0x00..0x7E).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e == 0 ? __fmul_rn((float)m, 0.001953125f) : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// One 16-element group with tensor scale g (g6 = fp32(6 g)):
//   s = amax / g6; sf = E4M3(s); d = dec(sf) * g; code_i = E2M1(a_i / d) (signed zero if
//   d == 0); deq_i = val(code_i) * d.
// Returns the scale byte; packs codes (element 2j low nibble of byte j) into lo/hi words.
__device__ __forceinline__ uint32_t nvfp4_group(const float (&a)[16], float g, float g6, uint32_t& lo, uint32_t& hi,
                                                float (&deq)[16]) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(a[i]));
    const float s = __fdiv_rn(amax, g6);
    const uint32_t sf = e4m3_encode_nonneg(s);
    const float d = __fmul_rn(e4m3_value(sf), g);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        uint32_t c;
        if (d > 0.0f) c = e2m1_encode(__fdiv_rn(a[i], d));
        else c = (__float_as_uint(a[i]) >> 28) & 8u;
        const float mag = __fmul_rn(e2m1_mag(c & 7u), d);
        deq[i] = (c & 8u) ? -mag : mag;
        w[i >> 3] |= c << (4 * (i & 7));
    }
    lo = w[0];
    hi = w[1];
    return sf;
}

// Byte offset of (row r, group q) in the GEMM's tiled scale layout of a matrix with
// `cols` columns: 512-byte chunks per (128-row tile, 4 groups), (t%32)*16 + (t/32)*4 + q%4.
__device__ __forceinline__ int64_t sf_swz_offset(int64_t r, int64_t q, int cols) {
    const int64_t ks = cols / 64, t = r & 127;
    return (((r >> 7) * ks + (q >> 2)) << 9) + ((t & 31) << 4) + ((t >> 5) << 2) + (q & 3);
}

}  // namespace mq

// Helpers shared by the quantization kernels (quant.cu) and the fused quantize +
// Delta-score kernel (select.cu), which in the whole-path call also quantizes the
// activation rows.
#pragma once

#include <cstdint>

#include "common.cuh"
#include "nvfp4.cuh"

namespace mq {

// Number of CTAs (and partial maxima) of the |W| maximum pass.
constexpr int kAmaxBlocks = 148;

// 16 bf16 values (32 bytes, 16-byte aligned) widened to fp32.
__device__ __forceinline__ void load16_bf16(const uint16_t* p, float (&a)[16]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    const uint4 v0 = __ldg(q), v1 = __ldg(q + 1);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        a[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        a[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
}

// Tensor scale from the kAmaxBlocks partial maxima: g = amax / 2688, or 1 for an
// all-zero tensor. Every thread of the CTA gets it (one shared-memory broadcast).
__device__ __forceinline__ float tensor_scale(const float* partial) {
    __shared__ float s_g;
    if (threadIdx.x < 32) {
        float m = 0.0f;
        for (int i = threadIdx.x; i < kAmaxBlocks; i += 32) m = fmaxf(m, __ldg(partial + i));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (threadIdx.x == 0) s_g = (m == 0.0f) ? 1.0f : __fdiv_rn(m, 2688.0f);
    }
    __syncthreads();
    return s_g;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Gathers the scale bytes of 4 consecutive groups (lanes l..l+3, l % 4 == 0) into one
// 32-bit word for lane l.
__device__ __forceinline__ uint32_t gather4(uint32_t b) {
    const uint32_t b1 = __shfl_down_sync(0xffffffffu, b, 1);
    const uint32_t b2 = __shfl_down_sync(0xffffffffu, b, 2);
    const uint32_t b3 = __shfl_down_sync(0xffffffffu, b, 3);
    return b | (b1 << 8) | (b2 << 16) | (b3 << 24);
}

// A6: token row m (of the M rows padded to a multiple of 128) by one whole CTA, every
// group held in registers (kGPT groups per thread, groups tid + j * blockDim), so the row
// is read once. Rows >= M only clear their tiled scales.
template <int kGPT>
__device__ __forceinline__ void quant_act_row(const uint16_t* __restrict__ X, int M, int K,
                                              uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                              uint8_t* __restrict__ sf_swz, float* __restrict__ g_x, int m) {
    const int G = K / 16;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (m >= M) {
        for (int q = threadIdx.x * 4; q < G; q += blockDim.x * 4)
            *reinterpret_cast<uint32_t*>(sf_swz + sf_swz_offset(m, q, K)) = 0u;
        return;
    }
    const uint16_t* row = X + (int64_t)m * K;
    float a[kGPT][16];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < kGPT; ++j) {
        const int q = threadIdx.x + j * blockDim.x;
        if (q < G) {
            load16_bf16(row + q * 16, a[j]);
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(a[j][i]));
        }
    }
    __shared__ float red[32];
    __shared__ float s_g;
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    if (warp == 0) {
        float t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
        t = warp_max(t);
        if (lane == 0) {
            s_g = (t == 0.0f) ? 1.0f : __fdiv_rn(t, 2688.0f);
            g_x[m] = s_g;
        }
    }
    __syncthreads();
    const float g = s_g, g6 = __fmul_rn(6.0f, g);
#pragma unroll
    for (int j = 0; j < kGPT; ++j) {
        const int q = threadIdx.x + j * blockDim.x;
        const bool live = q < G;
        uint32_t sfb = 0;
        if (live) {
            float deq[16];
            uint32_t lo, hi;
            sfb = nvfp4_group(a[j], g, g6, lo, hi, deq);
            reinterpret_cast<uint2*>(codes + (int64_t)m * (K / 2))[q] = make_uint2(lo, hi);
            if (sf) sf[(int64_t)m * G + q] = (uint8_t)sfb;
        }
        const uint32_t word = gather4(sfb);
        if (live && (lane & 3) == 0) *reinterpret_cast<uint32_t*>(sf_swz + sf_swz_offset(m, q, K)) = word;
    }
}

cudaError_t launch_amax(const uint16_t* W, int64_t n, float* partial, cudaStream_t s);

}  // namespace mq

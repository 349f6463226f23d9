// Helpers shared by the quantization kernels (quant.cu) and the fused quantize +
// Delta-score kernel (select.cu).
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

cudaError_t launch_amax(const uint16_t* W, int64_t n, float* partial, cudaStream_t s);

}  // namespace mq

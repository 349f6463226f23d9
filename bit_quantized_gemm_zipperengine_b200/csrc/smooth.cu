// Equivalent transform ahead of quantization (MosaicQuant summary, "Methodology",
// section 1: activation outliers are migrated into the weights by an equivalent transform
// such as SmoothQuant before the weight is split into base and residual). SmoothQuant's
// per-input-channel rule with migration strength 1/2:
//   s_k = sqrt(max_t |Xcal[t][k]| / max_n |W[n][k]|)   (1 if either maximum is 0),
//   W' = W diag(s), X' = X diag(s)^-1, so X W^T = X' W'^T up to the bf16 roundings.
// Every step is one IEEE fp32 operation (maximum, division, square root, multiply or
// divide, then the bf16 rounding), so the results match the CPU oracle bit for bit.
#include <cuda_bf16.h>

#include "common.cuh"
#include "nvfp4.cuh"

namespace mq {

namespace {

constexpr int kCols = 32;      // columns per CTA of the maxima kernel
constexpr int kThreads = 256;  // 8 warps; a warp covers 8 rows x 32 columns per step

// Maximum of |A[r][c0..c0+31]| over rows, per column, for this thread's 8 columns
// (thread t: column group t % 4, rows t / 4, t / 4 + 64, ...).
__device__ __forceinline__ void colmax8(const uint16_t* __restrict__ A, int rows, int K, int c0, float (&m)[8]) {
    const int t = threadIdx.x, g = t & 3;
    for (int r = t >> 2; r < rows; r += kThreads / 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(A + (int64_t)r * K + c0 + 8 * g));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            m[2 * j] = fmaxf(m[2 * j], fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)));
            m[2 * j + 1] = fmaxf(m[2 * j + 1], fabsf(bf16_bits_to_f32(w[j] >> 16)));
        }
    }
}

// The 8 maxima of every thread with the same column group, combined over the CTA; column
// c0 + 8g + j's maximum lands in out[8g + j].
__device__ __forceinline__ void combine(float (&m)[8], float* red, float* out) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], o));
    if (lane < 4)
#pragma unroll
        for (int j = 0; j < 8; ++j) red[(warp * 4 + lane) * 8 + j] = m[j];
    __syncthreads();
    if (t < kCols) {
        const int g = t >> 3, j = t & 7;
        float v = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w) v = fmaxf(v, red[(w * 4 + g) * 8 + j]);
        out[t] = v;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kThreads) k_smooth_scales(const uint16_t* __restrict__ Xcal, int T,
                                                           const uint16_t* __restrict__ W, int N, int K,
                                                           float* __restrict__ s) {
    __shared__ float red[kThreads / 32 * 4 * 8];
    __shared__ float ax[kCols], aw[kCols];
    griddep_wait();
    griddep_launch();
    const int c0 = blockIdx.x * kCols;
    float m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = 0.0f;
    colmax8(Xcal, T, K, c0, m);
    combine(m, red, ax);
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = 0.0f;
    colmax8(W, N, K, c0, m);
    combine(m, red, aw);
    if (threadIdx.x < kCols) {
        const float x = ax[threadIdx.x], w = aw[threadIdx.x];
        s[c0 + threadIdx.x] = (x == 0.0f || w == 0.0f) ? 1.0f : __fsqrt_rn(__fdiv_rn(x, w));
    }
}

// out = bf16(a * s_k) or bf16(a / s_k), eight elements per thread and step.
__global__ void __launch_bounds__(kThreads) k_smooth_apply(const uint16_t* __restrict__ A, int64_t n8, int K,
                                                          const float* __restrict__ s, int invert,
                                                          uint16_t* __restrict__ out) {
    griddep_wait();
    griddep_launch();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const int k0 = (int)((i * 8) % K);
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(A) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a0 = bf16_bits_to_f32(w[j] & 0xFFFFu), a1 = bf16_bits_to_f32(w[j] >> 16);
            const float s0 = __ldg(s + k0 + 2 * j), s1 = __ldg(s + k0 + 2 * j + 1);
            const float r0 = invert ? __fdiv_rn(a0, s0) : __fmul_rn(a0, s0);
            const float r1 = invert ? __fdiv_rn(a1, s1) : __fmul_rn(a1, s1);
            const __nv_bfloat16 b0 = __float2bfloat16_rn(r0), b1 = __float2bfloat16_rn(r1);
            o[j] = (uint32_t)(*reinterpret_cast<const uint16_t*>(&b0)) |
                   ((uint32_t)(*reinterpret_cast<const uint16_t*>(&b1)) << 16);
        }
        reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

cudaError_t launch_smooth_scales(const uint16_t* Xcal, int T, const uint16_t* W, int N, int K, float* s,
                                 cudaStream_t st) {
    return launch_pdl(k_smooth_scales, dim3(K / kCols), dim3(kThreads), 0, st, 1, Xcal, T, W, N, K, s);
}

cudaError_t launch_smooth_apply(const uint16_t* A, int rows, int K, const float* s, int invert, uint16_t* out,
                                cudaStream_t st) {
    const int64_t n8 = (int64_t)rows * K / 8;
    const int64_t want = (n8 + kThreads - 1) / kThreads;
    const int grid = (int)(want < 148 * 8 ? want : 148 * 8);
    return launch_pdl(k_smooth_apply, dim3(grid), dim3(kThreads), 0, st, 1, A, n8, K, s, invert, out);
}

}  // namespace mq

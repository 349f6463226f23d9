// Weight and activation quantization to NVFP4 (the dense 4-bit base and the 4-bit
// residual of MosaicQuant, summary "Methodology" section 1) and the diagonal Hessian
// estimate (section 2). HBM-bound elementwise kernels: 16-byte vector loads, one
// thread per 16-element group, warp-shuffle maxima.
#include "common.cuh"
#include "nvfp4.cuh"

namespace mq {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ void load16_bf16(const uint16_t* p, float (&a)[16]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    uint4 v0 = __ldg(q), v1 = __ldg(q + 1);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        a[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        a[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
}

// Per-CTA maxima of |W| over a grid-stride range of 8-element vectors.
__global__ void __launch_bounds__(256) k_amax_partial(const uint16_t* __restrict__ W, int64_t n8,
                                                      float* __restrict__ partial) {
    float m = 0.0f;
    const uint4* v = reinterpret_cast<const uint4*>(W);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        uint4 x = __ldg(v + i);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            m = fmaxf(m, fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)));
            m = fmaxf(m, fabsf(bf16_bits_to_f32(w[j] >> 16)));
        }
    }
    __shared__ float red[8];
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        t = warp_max(t);
        if (threadIdx.x == 0) partial[blockIdx.x] = t;
    }
}

// Tensor scale from the partial maxima: g = amax / 2688, or 1 for an all-zero tensor.
__device__ __forceinline__ float reduce_scale(const float* partial, int P) {
    __shared__ float s_g;
    if (threadIdx.x < 32) {
        float m = 0.0f;
        for (int i = threadIdx.x; i < P; i += 32) m = fmaxf(m, partial[i]);
        m = warp_max(m);
        if (threadIdx.x == 0) s_g = (m == 0.0f) ? 1.0f : __fdiv_rn(m, 2688.0f);
    }
    __syncthreads();
    return s_g;
}

// Gathers the scale bytes of 4 consecutive groups (lanes l..l+3, l % 4 == 0) into one
// 32-bit word for lane l.
__device__ __forceinline__ uint32_t gather4(uint32_t b) {
    const uint32_t b1 = __shfl_down_sync(0xffffffffu, b, 1);
    const uint32_t b2 = __shfl_down_sync(0xffffffffu, b, 2);
    const uint32_t b3 = __shfl_down_sync(0xffffffffu, b, 3);
    return b | (b1 << 8) | (b2 << 16) | (b3 << 24);
}

// A1: base NVFP4(W, g) and residual NVFP4(W - deq Q(W), g) for every group.
// One thread per group; the group count is a multiple of 32 (K % 64 == 0 gives
// K/16 % 4 == 0 and N*K/16 % 32 == 0 needs N % 8 == 0, true for N % 64 == 0).
__global__ void __launch_bounds__(256) k_quant_weight(const uint16_t* __restrict__ W, int N, int K,
                                                      const float* __restrict__ partial, int P,
                                                      uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                      uint8_t* __restrict__ sf_swz, float* __restrict__ g_out,
                                                      uint8_t* __restrict__ rcodes, uint8_t* __restrict__ rsf) {
    const float g = reduce_scale(partial, P);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
    const float g6 = __fmul_rn(6.0f, g);
    const int G = K / 16;
    const int64_t ngrp = (int64_t)N * G;
    const int lane = threadIdx.x & 31;
    for (int64_t grp = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; grp - lane < ngrp;
         grp += (int64_t)gridDim.x * blockDim.x) {
        const bool live = grp < ngrp;
        float a[16], deq[16];
        uint32_t lo = 0, hi = 0, sfb = 0;
        if (live) {
            load16_bf16(W + grp * 16, a);
            sfb = nvfp4_group(a, g, g6, lo, hi, deq);
            reinterpret_cast<uint2*>(codes)[grp] = make_uint2(lo, hi);
            if (sf) sf[grp] = (uint8_t)sfb;
        }
        const uint32_t word = gather4(sfb);
        if (live && (lane & 3) == 0) {
            const int64_t r = grp / G, q = grp % G;
            *reinterpret_cast<uint32_t*>(sf_swz + sf_swz_offset(r, q, K)) = word;
        }
        if (live) {
            float R[16], rdeq[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) R[i] = __fsub_rn(a[i], deq[i]);
            uint32_t rlo, rhi;
            const uint32_t rs = nvfp4_group(R, g, g6, rlo, rhi, rdeq);
            reinterpret_cast<uint2*>(rcodes)[grp] = make_uint2(rlo, rhi);
            rsf[grp] = (uint8_t)rs;
        }
    }
}

// A6: one CTA per (padded) token row. Rows >= M only clear their tiled scales.
__global__ void __launch_bounds__(128) k_quant_act(const uint16_t* __restrict__ X, int M, int K,
                                                   uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                   uint8_t* __restrict__ sf_swz, float* __restrict__ g_x) {
    const int m = blockIdx.x;
    const int G = K / 16;
    const int lane = threadIdx.x & 31;
    if (m >= M) {
        for (int q = threadIdx.x * 4; q < G; q += blockDim.x * 4)
            *reinterpret_cast<uint32_t*>(sf_swz + sf_swz_offset(m, q, K)) = 0u;
        return;
    }
    const uint16_t* row = X + (int64_t)m * K;
    float amax = 0.0f;
    for (int q = threadIdx.x; q < G; q += blockDim.x) {
        float a[16];
        load16_bf16(row + q * 16, a);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(a[i]));
    }
    __shared__ float red[4];
    __shared__ float s_g;
    amax = warp_max(amax);
    if (lane == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        s_g = (t == 0.0f) ? 1.0f : __fdiv_rn(t, 2688.0f);
        g_x[m] = s_g;
    }
    __syncthreads();
    const float g = s_g, g6 = __fmul_rn(6.0f, g);
    // G is a multiple of 4; iterate whole warps so the 4-group gather stays aligned.
    for (int q0 = (threadIdx.x & ~31); q0 < G; q0 += blockDim.x) {
        const int q = q0 + lane;
        const bool live = q < G;
        uint32_t sfb = 0;
        if (live) {
            float a[16], deq[16];
            uint32_t lo, hi;
            load16_bf16(row + q * 16, a);
            sfb = nvfp4_group(a, g, g6, lo, hi, deq);
            reinterpret_cast<uint2*>(codes + (int64_t)m * (K / 2))[q] = make_uint2(lo, hi);
            if (sf) sf[(int64_t)m * G + q] = (uint8_t)sfb;
        }
        const uint32_t word = gather4(sfb);
        if (live && (lane & 3) == 0) *reinterpret_cast<uint32_t*>(sf_swz + sf_swz_offset(m, q, K)) = word;
    }
}

// A2: H_k = fp32( sum_t x_tk^2 / T ) with the fp64 sum taken in t order (one thread per
// column; the squares of bf16 values are exact in fp64, so a fused add is harmless).
__global__ void __launch_bounds__(128) k_hessian(const uint16_t* __restrict__ X, int T, int K, float* __restrict__ H) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    double s = 0.0;
    int t = 0;
    for (; t + 8 <= T; t += 8) {
        uint16_t v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __ldg(X + (int64_t)(t + j) * K + k);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const double x = (double)bf16_bits_to_f32(v[j]);
            s = __dadd_rn(s, __dmul_rn(x, x));
        }
    }
    for (; t < T; ++t) {
        const double x = (double)bf16_bits_to_f32(__ldg(X + (int64_t)t * K + k));
        s = __dadd_rn(s, __dmul_rn(x, x));
    }
    H[k] = __double2float_rn(__ddiv_rn(s, (double)T));
}

// ------------------------------------------------------------------ launchers
int amax_grid(int64_t n8) {
    int64_t blocks = (n8 + 255) / 256;
    return (int)(blocks < 148 * 8 ? (blocks < 1 ? 1 : blocks) : 148 * 8);
}

cudaError_t launch_quant_weight(const uint16_t* W, int N, int K, uint8_t* codes, uint8_t* sf, uint8_t* sf_swz,
                                float* g, uint8_t* rcodes, uint8_t* rsf, float* partial, cudaStream_t s) {
    const int64_t n8 = (int64_t)N * K / 8;
    const int P = amax_grid(n8);
    k_amax_partial<<<P, 256, 0, s>>>(W, n8, partial);
    const int64_t ngrp = (int64_t)N * (K / 16);
    int64_t blocks = (ngrp + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_quant_weight<<<(int)blocks, 256, 0, s>>>(W, N, K, partial, P, codes, sf, sf_swz, g, rcodes, rsf);
    return cudaGetLastError();
}

cudaError_t launch_quant_act(const uint16_t* X, int M, int K, uint8_t* codes, uint8_t* sf, uint8_t* sf_swz,
                             float* g, cudaStream_t s) {
    const int Mp = (M + 127) / 128 * 128;
    k_quant_act<<<Mp, 128, 0, s>>>(X, M, K, codes, sf, sf_swz, g);
    return cudaGetLastError();
}

cudaError_t launch_hessian(const uint16_t* X, int T, int K, float* H, cudaStream_t s) {
    k_hessian<<<(K + 127) / 128, 128, 0, s>>>(X, T, K, H);
    return cudaGetLastError();
}

}  // namespace mq

// Weight and activation quantization to NVFP4 (the dense 4-bit base and the 4-bit
// residual of MosaicQuant, summary "Methodology" section 1) and the diagonal Hessian
// estimate (section 2). HBM-bound elementwise kernels: 16-byte vector loads, one
// thread per 16-element group, warp-shuffle maxima, hardware E2M1 conversions.
#include "common.cuh"
#include "nvfp4.cuh"
#include "quant.cuh"

namespace mq {

// 16-byte read-only streaming load (not kept in L1).
__device__ __forceinline__ uint4 ld_stream16(const uint4* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// ld_stream16 with an L2 cache policy.
__device__ __forceinline__ uint4 ld_stream16_hint(const uint4* p, uint64_t policy) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p), "l"(policy));
    return r;
}

// Per-CTA maxima of |W| over a grid-stride range of 8-element vectors (kAmaxBlocks
// CTAs of 512 threads, 8 independent 16-byte loads in flight per thread: 64 KB per SM,
// about what HBM needs in flight to run at full rate).
// W is an input of the call, never written by the preceding kernel, so the kernel lets
// its dependent start and reads W at once: it overlaps the preceding kernel (the Hessian
// estimate, which it does not use). It waits for that kernel only at its end, so that
// its own completion still implies the predecessor's. The partials it overwrites are
// read by the quantizers before they let their dependents start.
__global__ void __launch_bounds__(512, 1) k_amax_partial(const uint16_t* __restrict__ W, int64_t n8,
                                                      float* __restrict__ partial) {
    griddep_launch();
    float m = 0.0f;
    const uint4* v = reinterpret_cast<const uint4*>(W);
    // W is read again right after by the quantize+Delta pass: keep it in L2 until then
    const uint64_t keep = l2_policy_evict_last();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    for (; i < n8; i += 8 * stride) {
        uint4 x[8];
        // volatile: the eight loads are issued before any of them is used. In the last
        // round an index past the end reads the last vector again (a repeated element does
        // not change the maximum), so the remainder also goes out eight loads at a time.
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t j = i + u * stride;
            x[u] = ld_stream16_hint(v + (j < n8 ? j : n8 - 1), keep);
        }
        // every loaded word is an operand here, so all eight loads precede the first use
        asm volatile("" : "+r"(x[0].x), "+r"(x[0].y), "+r"(x[0].z), "+r"(x[0].w), "+r"(x[1].x), "+r"(x[1].y),
                     "+r"(x[1].z), "+r"(x[1].w), "+r"(x[2].x), "+r"(x[2].y), "+r"(x[2].z), "+r"(x[2].w),
                     "+r"(x[3].x), "+r"(x[3].y), "+r"(x[3].z), "+r"(x[3].w));
        asm volatile("" : "+r"(x[4].x), "+r"(x[4].y), "+r"(x[4].z), "+r"(x[4].w), "+r"(x[5].x), "+r"(x[5].y),
                     "+r"(x[5].z), "+r"(x[5].w), "+r"(x[6].x), "+r"(x[6].y), "+r"(x[6].z), "+r"(x[6].w),
                     "+r"(x[7].x), "+r"(x[7].y), "+r"(x[7].z), "+r"(x[7].w));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)),
                                                           fabsf(bf16_bits_to_f32(w[j] >> 16))));
        }
    }
    __shared__ float red[16];
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        t = warp_max(t);
        if (threadIdx.x == 0) partial[blockIdx.x] = t;
    }
    griddep_wait();
}

// A1: base NVFP4(W, g) and residual NVFP4(W - deq Q(W), g) for every group.
// One thread per group; the group count is a multiple of 32 (K % 64 == 0 and
// N % 64 == 0), so whole warps stay together for the 4-group scale gather. The groups of
// the rows past N up to the next multiple of 128 write zero tiled scales.
__global__ void __launch_bounds__(256) k_quant_weight(const uint16_t* __restrict__ W, int N, int K,
                                                      const float* __restrict__ partial,
                                                      uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                      uint8_t* __restrict__ sf_swz, float* __restrict__ g_out,
                                                      uint8_t* __restrict__ rcodes, uint8_t* __restrict__ rsf) {
    griddep_wait();
    const float g = tensor_scale(partial);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
    griddep_launch();  // once every CTA has read the partials
    const float g6 = __fmul_rn(6.0f, g);
    const int G = K / 16;
    const int64_t ngrp = (int64_t)N * G;
    const int64_t ngrp_pad = (int64_t)((N + 127) / 128 * 128) * G;  // rows past N: zero tiled scales
    const int lane = threadIdx.x & 31;
    for (int64_t grp = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; grp - lane < ngrp_pad;
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
        if (grp < ngrp_pad && (lane & 3) == 0) {
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

// early == 0: wait for the preceding kernel, let the dependent start, quantize.
// early != 0: let the dependent start, quantize, then wait for the preceding kernel before
// exiting (so this kernel's completion still implies its predecessor's). For a caller
// whose X and outputs are not touched by the kernels still running before it.
template <int kGPT>
__global__ void __launch_bounds__(1024)
    k_quant_act(const uint16_t* __restrict__ X, int M, int K, uint8_t* __restrict__ codes,
                uint8_t* __restrict__ sf, uint8_t* __restrict__ sf_swz, float* __restrict__ g_x, int early) {
    if (!early) griddep_wait();
    griddep_launch();
    quant_act_row<kGPT>(X, M, K, codes, sf, sf_swz, g_x, blockIdx.x);
    if (early) griddep_wait();
}

// A2: H_k = fp32(S_k / T), S_k the fp64 sum of the exact squares fp64(x_tk)^2 by a fixed
// pairwise tree over t: the squares padded with zeros to a power of two P >= T, then
// v[i] += v[i + h] for h = P/2, ..., 1. Every sum in the tree is >= +0 and x + (+0) == x,
// so the padding leaves change nothing and any power of two >= T gives the same S_k; the
// kernel takes P = 512 * NB (NB = 1 for T <= 512, 2 for T <= 1024).
// A CTA of 8 warps owns 32 columns; lane l of warp w holds the rows i = r0 + 64 j with
// r0 = 8 (l >> 2) + w and the 8 columns of quad l & 3 (one 16-byte load per row, 64
// contiguous bytes per row per warp). The tree's levels, in order:
//   h = P/2 .. 64  rows of one thread: J = 8 NB leaves j, taken as NB batches of 8
//                  (batch b: j = b + NB m), each the 8-leaf tree over m, then the batches;
//   h = 32, 16, 8  lanes 16, 8, 4 apart (r0 + 32, + 16, + 8);
//   h = 4, 2, 1    warps, in shared memory, one thread per column.
constexpr int kHMaxTokens = 1024;
template <int NB>
__global__ void __launch_bounds__(256) k_hessian(const uint16_t* __restrict__ X, int T, int K,
                                                 float* __restrict__ H) {
    griddep_wait();
    griddep_launch();
    __shared__ double red[8][33];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = 8 * (lane >> 2) + w, c0 = blockIdx.x * 32 + (lane & 3) * 8;
    uint4 raw[8 * NB];
#pragma unroll
    for (int j = 0; j < 8 * NB; ++j) {
        const int i = r0 + 64 * j;
        raw[j] = i < T ? ld_stream16(reinterpret_cast<const uint4*>(X + (int64_t)i * K + c0)) : make_uint4(0, 0, 0, 0);
    }
    double acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            double u[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const uint4 r = raw[b + NB * m];
                const uint32_t wd = c < 2 ? r.x : c < 4 ? r.y : c < 6 ? r.z : r.w;
                const double x = (double)bf16_bits_to_f32((c & 1) ? wd >> 16 : wd & 0xFFFFu);
                u[m] = __dmul_rn(x, x);
            }
#pragma unroll
            for (int h = 4; h >= 1; h >>= 1)
#pragma unroll
                for (int m = 0; m < h; ++m) u[m] = __dadd_rn(u[m], u[m + h]);
            acc[c] = b == 0 ? u[0] : __dadd_rn(acc[c], u[0]);
        }
    }
#pragma unroll
    for (int h = 16; h >= 4; h >>= 1)  // lanes below h end with the sums they need
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = __dadd_rn(acc[c], __shfl_down_sync(0xFFFFFFFFu, acc[c], h));
    if (lane < 4)
#pragma unroll
        for (int c = 0; c < 8; ++c) red[w][lane * 8 + c] = acc[c];
    __syncthreads();
    if (w == 0) {
        double u[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) u[m] = red[m][lane];
#pragma unroll
        for (int h = 4; h >= 1; h >>= 1)
#pragma unroll
            for (int m = 0; m < h; ++m) u[m] = __dadd_rn(u[m], u[m + h]);
        H[blockIdx.x * 32 + lane] = __double2float_rn(__ddiv_rn(u[0], (double)T));
    }
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_amax(const uint16_t* W, int64_t n, float* partial, cudaStream_t s) {
    return launch_pdl(k_amax_partial, dim3(kAmaxBlocks), dim3(512), 0, s, 1, W, n / 8, partial);
}

cudaError_t launch_quant_weight(const uint16_t* W, int N, int K, uint8_t* codes, uint8_t* sf, uint8_t* sf_swz,
                                float* g, uint8_t* rcodes, uint8_t* rsf, float* partial, cudaStream_t s) {
    cudaError_t e = launch_amax(W, (int64_t)N * K, partial, s);
    if (e != cudaSuccess) return e;
    const int64_t ngrp = (int64_t)N * (K / 16);
    int64_t blocks = (ngrp + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return launch_pdl(k_quant_weight, dim3((unsigned)blocks), dim3(256), 0, s, 1, W, N, K, (const float*)partial,
                      codes, sf, sf_swz, g, rcodes, rsf);
}

cudaError_t launch_quant_act(const uint16_t* X, int M, int K, uint8_t* codes, uint8_t* sf, uint8_t* sf_swz,
                             float* g, bool early, cudaStream_t s) {
    const int Mp = (M + 127) / 128 * 128;
    const int G = K / 16;
    const int gpt = G <= 1024 ? 1 : G <= 2048 ? 2 : 4;
    if (G > 4 * 1024) return cudaErrorInvalidValue;
    int threads = (G + gpt - 1) / gpt;
    threads = (threads + 31) / 32 * 32;
    const int e = early ? 1 : 0;
    if (gpt == 1)
        return launch_pdl(k_quant_act<1>, dim3(Mp), dim3(threads), 0, s, 1, X, M, K, codes, sf, sf_swz, g, e);
    if (gpt == 2)
        return launch_pdl(k_quant_act<2>, dim3(Mp), dim3(threads), 0, s, 1, X, M, K, codes, sf, sf_swz, g, e);
    return launch_pdl(k_quant_act<4>, dim3(Mp), dim3(threads), 0, s, 1, X, M, K, codes, sf, sf_swz, g, e);
}

cudaError_t launch_hessian(const uint16_t* X, int T, int K, float* H, cudaStream_t s) {
    if (T > 512) return launch_pdl(k_hessian<2>, dim3(K / 32), dim3(256), 0, s, 1, X, T, K, H);
    return launch_pdl(k_hessian<1>, dim3(K / 32), dim3(256), 0, s, 1, X, T, K, H);
}

int hessian_max_tokens() { return kHMaxTokens; }

}  // namespace mq

// The dense FP4 tensor-core rate of this GPU, measured: every CTA keeps one A tile
// (128 x 256 K E2M1), one B tile (256 x 256 K) and their E4M3 scales resident in shared
// and tensor memory and issues back-to-back tcgen05.mma kind::mxf4nvf4 (M = 128,
// N = 256, K = 64) into one fp32 accumulator, with no loads in the loop. The roofline
// fractions of the fused GEMM's large-M kernel are taken against this rate.
#include "common.cuh"
#include "mosaic_probe.h"

namespace mq {

cudaError_t error_word(int** ptr);

namespace {

constexpr int kOffA = 0;            // 128 rows x 128 B (swizzled), 4 K steps of 64
constexpr int kOffB = 16384;        // 256 rows x 128 B (swizzled)
constexpr int kOffSFA = 49152;      // 4 chunks x 512 B
constexpr int kOffSFB = 51200;      // 2 row tiles x 4 chunks x 512 B
constexpr int kOffBar = 55296;
constexpr int kSmem = kOffBar + 64 + 1024;

__global__ void __launch_bounds__(128, 1) k_fp4_mma_loop(int iters, int* err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* done = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
    const int warp = threadIdx.x >> 5;
    // operands: a fixed pseudo-random byte pattern (both signs, every E2M1 magnitude);
    // scales 1.0 (E4M3 0x38), so the accumulator stays finite
    for (int i = threadIdx.x; i < kOffSFA / 4; i += blockDim.x) {
        uint32_t h = (uint32_t)i * 2654435761u + (uint32_t)blockIdx.x * 40503u;
        h ^= h >> 15;
        reinterpret_cast<uint32_t*>(smem)[i] = h * 2246822519u;
    }
    for (int i = threadIdx.x; i < (kOffBar - kOffSFA) / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(smem + kOffSFA)[i] = 0x38383838u;
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t sb = smem_u32(smem);
    if (threadIdx.x == 0) {
        const uint32_t sfa = tmem + 256, sfb = tmem + 272;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            tc_cp_sf_chunk(sfa + 4 * kk, smem_desc(sb + kOffSFA + kk * 512, 0, 128, 0));
            tc_cp_sf_chunk(sfb + 8 * kk, smem_desc(sb + kOffSFB + kk * 512, 0, 128, 0));
            tc_cp_sf_chunk(sfb + 8 * kk + 4, smem_desc(sb + kOffSFB + 2048 + kk * 512, 0, 128, 0));
        }
        constexpr uint32_t idesc = idesc_mxf4nvf4(128, 256);
        for (int i = 0; i < iters; ++i) {
            const int kk = i & 3;
            mma_mxf4nvf4(tmem, smem_desc(sb + kOffA + 32 * kk, 16, 1024, 2), smem_desc(sb + kOffB + 32 * kk, 16, 1024, 2),
                         idesc, sfa + 4 * kk, sfb + 8 * kk, i > 0 ? 1u : 0u);
        }
        tc_commit(done);
        // bounded wait (2 s) for the last MMA
        if (!mbar_try_wait(done, 0)) {
            const unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(done, 0))
                if (globaltimer_ns() - t0 > 2000000000ull) {
                    atomicCAS(err, 0, (int)MQ_ERR_TIMEOUT);
                    break;
                }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace
}  // namespace mq

extern "C" {

double mq_fp4_mma_loop_flops(int ctas, int iters) { return (double)ctas * iters * 2.0 * 128 * 256 * 64; }

mq_status mq_fp4_mma_loop(int ctas, int iters, mq_stream stream) {
    using namespace mq;
    if (ctas <= 0 || iters <= 0 || iters > (1 << 24)) return MQ_ERR_INVALID_ARG;
    static std::atomic<bool> attr_set[64];
    if (once_per_device(attr_set, [] {
            return cudaFuncSetAttribute(k_fp4_mma_loop, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        }) != cudaSuccess)
        return MQ_ERR_CUDA;
    int* err = nullptr;
    if (error_word(&err) != cudaSuccess) return MQ_ERR_CUDA;
    k_fp4_mma_loop<<<ctas, 128, kSmem, reinterpret_cast<cudaStream_t>(stream)>>>(iters, err);
    return cudaGetLastError() == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}

}  // extern "C"

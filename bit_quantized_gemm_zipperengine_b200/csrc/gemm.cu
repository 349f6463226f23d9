// ZipperEngine fused GEMM on sm_100a (MosaicQuant summary, "Methodology" section 3;
// arXiv 2606.15652 abstract: sparse block computation fused into the dense 4-bit GEMM
// through an overlapped pipeline).
//
// Decode kernel (small M): the weight is the MMA's M side (128 weight rows per tile),
// tokens are its N side (BN = 16..128), so a tile streams 128 x K of W exactly once.
// Warp roles: warp 0 issues TMA / bulk copies, warp 1 owns tensor memory and issues
// tcgen05 MMAs from one thread, warps 2-5 run the epilogue. Per K stage (256 K
// elements) the producer loads the W and X tiles (128-byte swizzle), their 4 scale
// chunks, and every selected residual block of the tile's two 64-row block rows.
// The MMA thread issues 4 base MMAs (K = 64 each) and one more MMA per selected
// residual block into the SAME fp32 accumulator: the residual block's rows fill one
// half of a 128-row operand whose other half carries zero scales. Split-K partials
// are added in a fixed order by the last CTA of each tile (a tile counter in the
// workspace), then scaled by g_x[m] * g_w and stored as bf16.
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.cuh"

namespace mq {

// Device error word (0 = fine, otherwise an mq_status); read and cleared by mq_get_error.
__device__ int g_error = 0;

// Wall-clock budget of a single pipeline wait before a kernel gives up (2 s).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for the phase with the given parity to complete. Gives up after kWaitLimitNs,
// records MQ_ERR_TIMEOUT in the device error word and returns false; the caller then
// stops issuing work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > kWaitLimitNs) {
            atomicCAS(&g_error, 0, (int)MQ_ERR_TIMEOUT);
            return false;
        }
    }
}

template <int BN>
struct DecodeCfg {
    static constexpr int kStages = BN >= 128 ? 3 : 4;
    static constexpr int kOffW = 0;                      // 128 rows x 128 B, swizzled
    static constexpr int kOffX = 16384;                  // BN rows x 128 B, swizzled
    static constexpr int kOffSFW = kOffX + BN * 128;     // 4 x 512 B
    static constexpr int kOffSFX = kOffSFW + 2048;       // 4 x 512 B
    static constexpr int kOffRC = kOffSFX + 2048;        // 4 x (128 rows x 32 B), no swizzle
    static constexpr int kOffRSF = kOffRC + 16384;       // 8 x 512 B
    static constexpr int kStageBytes = kOffRSF + 4096;
    static constexpr int kCtrlBytes = 256;
    static constexpr int kSmemBytes = kStages * kStageBytes + kCtrlBytes + 1024;
    static constexpr int kThreads = 192;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kSfCol0 = 128;                  // scale columns start after D
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Residual blocks of block row nt among block columns [kt0, kt0 + 4): returns a 4-bit
// presence mask and fills idx[kk] with the packed index of block (nt, kt0 + kk).
__device__ __forceinline__ uint32_t resid_lookup(const GemmParams& p, int nt, int kt0, int (&idx)[4]) {
    const int KB = p.K / 64, KW = (KB + 31) / 32;
    const uint32_t* row = p.bitmap + (int64_t)nt * KW;
    const int w = kt0 >> 5, sh = kt0 & 31;  // kt0 % 4 == 0, so the 4 bits share a word
    const uint32_t word = __ldg(row + w);
    const uint32_t m = (word >> sh) & 15u;
    if (m) {
        int base = __ldg(p.tile_ptr + nt);
        for (int j = 0; j < w; ++j) base += __popc(__ldg(row + j));
        base += __popc(sh ? (word & ((1u << sh) - 1u)) : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            idx[kk] = base;
            base += (m >> kk) & 1u;
        }
    }
    return m;
}

__device__ __forceinline__ bool tile_has_mma(const GemmParams& p, int n_tile, int ks_begin, int ks_end) {
    if (ks_end <= ks_begin) return false;
    if (p.mode != 2) return true;
    if (!p.has_resid) return false;
    for (int ks = ks_begin; ks < ks_end; ++ks)
        for (int h = 0; h < 2; ++h) {
            int idx[4];
            if (resid_lookup(p, n_tile * 2 + h, ks * 4, idx)) return true;
        }
    return false;
}

template <int BN>
__global__ void __launch_bounds__(192, 1)
    k_gemm_decode(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                  const GemmParams p) {
    using C = DecodeCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
    uint64_t* empty = full + C::kStages;
    uint64_t* accf = empty + C::kStages;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accf + 1);
    uint32_t* rmask = tmem_holder + 1;  // [kStages]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tile = blockIdx.x, split = blockIdx.y, m_tile = blockIdx.z;
    const int n0 = n_tile * 128, m0 = m_tile * BN;
    const int KS = p.K / 256, KS64 = p.K / 64;
    const int ks_begin = split * p.iters_per_split;
    const int ks_end = min(KS, ks_begin + p.iters_per_split);
    const int n_iters = max(0, ks_end - ks_begin);

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmap_w);
        tma_prefetch_desc(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ producer
            const uint8_t* xsf_tile = p.x_sf + (int64_t)(m0 / 128) * KS64 * 512;
            const uint8_t* wsf_tile = p.w_sf + (int64_t)n_tile * KS64 * 512;
            int issued = 0;
            for (int it = 0; it < n_iters; ++it) {
                const int s = it % C::kStages;
                const uint32_t use = it / C::kStages;
                if (it >= C::kStages && !mbar_wait(&empty[s], (use - 1) & 1)) break;
                const int ks = ks_begin + it;
                uint32_t m = 0;
                int idx0[4] = {0, 0, 0, 0}, idx1[4] = {0, 0, 0, 0};
                if (p.has_resid) {
                    const uint32_t m0b = resid_lookup(p, n_tile * 2 + 0, ks * 4, idx0);
                    const uint32_t m1b = resid_lookup(p, n_tile * 2 + 1, ks * 4, idx1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) m |= (((m0b >> kk) & 1u) << (2 * kk)) | (((m1b >> kk) & 1u) << (2 * kk + 1));
                }
                rmask[s] = m;
                uint8_t* st = smem + s * C::kStageBytes;
                const uint32_t bytes = 16384 + BN * 128 + 2048 + 2048 + __popc(m) * (2048 + 512);
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(st + C::kOffW, &tmap_w, &full[s], ks * 128, n0);
                tma_load_2d(st + C::kOffX, &tmap_x, &full[s], ks * 128, m0);
                bulk_load(st + C::kOffSFW, wsf_tile + (int64_t)ks * 4 * 512, 2048, &full[s]);
                bulk_load(st + C::kOffSFX, xsf_tile + (int64_t)ks * 4 * 512, 2048, &full[s]);
#pragma unroll 1
                for (int j = 0; j < 8; ++j) {
                    if (!((m >> j) & 1u)) continue;
                    const int kk = j >> 1, h = j & 1;
                    const int idx = h ? idx1[kk] : idx0[kk];
                    bulk_load(st + C::kOffRC + kk * 4096 + h * 2048, p.blk_codes + (int64_t)idx * 2048, 2048, &full[s]);
                    bulk_load(st + C::kOffRSF + j * 512, p.blk_sf + (int64_t)idx * 512, 512, &full[s]);
                }
                ++issued;
            }
            // Do not leave while copies into this CTA's shared memory are in flight.
            for (int it = max(0, issued - C::kStages); it < issued; ++it)
                mbar_wait(&full[it % C::kStages], (it / C::kStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_mxf4nvf4(128, BN);
            uint32_t acc = 0;
            for (int it = 0; it < n_iters; ++it) {
                const int s = it % C::kStages;
                const uint32_t use = it / C::kStages;
                if (!mbar_wait(&full[s], use & 1)) break;
                tc_fence_after();
                uint8_t* st = smem + s * C::kStageBytes;
                const uint32_t sfc = tmem + C::kSfCol0 + s * 64;
                const uint32_t m = rmask[s];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    tc_cp_sf_chunk(sfc + 4 * kk, smem_desc(smem_u32(st + C::kOffSFW + kk * 512), 0, 128, 0));
                    tc_cp_sf_chunk(sfc + 16 + 4 * kk, smem_desc(smem_u32(st + C::kOffSFX + kk * 512), 0, 128, 0));
                }
#pragma unroll 1
                for (int j = 0; j < 8; ++j)
                    if ((m >> j) & 1u)
                        tc_cp_sf_chunk(sfc + 32 + 4 * j, smem_desc(smem_u32(st + C::kOffRSF + j * 512), 0, 128, 0));
                const uint32_t aw = smem_u32(st + C::kOffW), bx = smem_u32(st + C::kOffX);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bdesc = smem_desc(bx + 32 * kk, 16, 1024, 2);
                    if (p.mode != 2) {
                        mma_mxf4nvf4(tmem, smem_desc(aw + 32 * kk, 16, 1024, 2), bdesc, idesc, sfc + 4 * kk,
                                     sfc + 16 + 4 * kk, acc);
                        acc = 1;
                    }
                    if (p.mode != 1) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int j = 2 * kk + h;
                            if (!((m >> j) & 1u)) continue;
                            const uint64_t adesc = smem_desc(smem_u32(st + C::kOffRC + kk * 4096), 128, 256, 0);
                            mma_mxf4nvf4(tmem, adesc, bdesc, idesc, sfc + 32 + 4 * j, sfc + 16 + 4 * kk, acc);
                            acc = 1;
                        }
                    }
                }
                tc_commit(&empty[s]);
            }
            tc_commit(accf);
        }
    } else {
        // ---------------------------------------------------- epilogue (warps 2..5)
        const int q = warp & 3;
        const int n = n0 + 32 * q + lane;
        float acc[BN];
        const bool waited = mbar_wait(accf, 0);
        tc_fence_after();
        if (waited && tile_has_mma(p, n_tile, ks_begin, ks_end)) {
#pragma unroll
            for (int c = 0; c < BN / 16; ++c) tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + 16 * c, acc + 16 * c);
        } else {
#pragma unroll
            for (int j = 0; j < BN; ++j) acc[j] = 0.0f;
        }
        tc_fence_before();
        const float gw = __ldg(p.g_w);
        if (p.splits == 1) {
#pragma unroll
            for (int j = 0; j < BN; ++j) {
                const int mm = m0 + j;
                if (mm < p.M) {
                    const float sc = __fmul_rn(__ldg(p.g_x + mm), gw);
                    const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(acc[j], sc));
                    p.Y[(int64_t)mm * p.N + n] = *reinterpret_cast<const uint16_t*>(&y);
                }
            }
        } else {
            const int Mp = gridDim.z * BN;
            float* part = p.partial + ((int64_t)split * Mp + m0) * p.N + n;
#pragma unroll
            for (int j = 0; j < BN; ++j) __stcg(part + (int64_t)j * p.N, acc[j]);
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            __shared__ int s_last;
            int* ctr = p.counters + m_tile * gridDim.x + n_tile;
            if (threadIdx.x == 64) s_last = (atomicAdd(ctr, 1) == p.splits - 1);
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (s_last) {
                __threadfence();
                const float* base = p.partial + (int64_t)m0 * p.N + n;
#pragma unroll 1
                for (int j = 0; j < BN; ++j) {
                    const int mm = m0 + j;
                    if (mm >= p.M) break;
                    float sum = __ldcg(base + (int64_t)j * p.N);
                    for (int s2 = 1; s2 < p.splits; ++s2)
                        sum = __fadd_rn(sum, __ldcg(base + ((int64_t)s2 * Mp + j) * p.N));
                    const float sc = __fmul_rn(__ldg(p.g_x + mm), gw);
                    const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(sum, sc));
                    p.Y[(int64_t)mm * p.N + n] = *reinterpret_cast<const uint16_t*>(&y);
                }
                if (threadIdx.x == 64) *ctr = 0;
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
DecodePlan plan_decode(int M, int N, int K) {
    DecodePlan d;
    d.BN = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
    d.tiles_m = (M + d.BN - 1) / d.BN;
    d.tiles_n = N / 128;
    const int KS = K / 256;
    const int tiles = d.tiles_m * d.tiles_n;
    int s = 148 / tiles;
    if (s < 1) s = 1;
    if (s > KS) s = KS;
    d.iters = (KS + s - 1) / s;
    d.splits = (KS + d.iters - 1) / d.iters;
    return d;
}

size_t decode_workspace_bytes(int M, int N, int K) {
    DecodePlan d = plan_decode(M, N, K);
    if (d.splits <= 1) return 0;
    size_t part = (size_t)d.splits * d.tiles_m * d.BN * N * sizeof(float);
    part = (part + 255) & ~size_t(255);
    return part + (size_t)d.tiles_m * d.tiles_n * sizeof(int);
}

template <int BN>
static cudaError_t launch_decode_bn(const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                                   const DecodePlan& d, cudaStream_t s) {
    using C = DecodeCfg<BN>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm_decode<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(d.tiles_n, d.splits, d.tiles_m);
    k_gemm_decode<BN><<<grid, C::kThreads, C::kSmemBytes, s>>>(tw, tx, p);
    return cudaGetLastError();
}

cudaError_t launch_gemm_decode(const CUtensorMap& tw, const CUtensorMap& tx, GemmParams p, const DecodePlan& d,
                               cudaStream_t s) {
    p.splits = d.splits;
    p.iters_per_split = d.iters;
    switch (d.BN) {
        case 16: return launch_decode_bn<16>(tw, tx, p, d, s);
        case 32: return launch_decode_bn<32>(tw, tx, p, d, s);
        case 64: return launch_decode_bn<64>(tw, tx, p, d, s);
        default: return launch_decode_bn<128>(tw, tx, p, d, s);
    }
}

cudaError_t read_clear_error(int* value) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_error, sizeof(int));
    if (e != cudaSuccess || *value == 0) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_error, &zero, sizeof(int));
}

}  // namespace mq

// ZipperEngine fused GEMM on sm_100a (MosaicQuant summary, "Methodology" section 3;
// arXiv 2606.15652 abstract: sparse block computation fused into the dense 4-bit GEMM
// through an overlapped pipeline). Base and residual blocks accumulate into one fp32
// tensor-memory accumulator (tcgen05 kind::mxf4nvf4, one extra MMA per selected block).
//
// Three kernels:
//  - k_gemm_streamk (small M, HBM-bound): the weight is the MMA's M side (128 weight rows
//    per tile), the tokens its N side; persistent CTAs take equal ranges of (tile,
//    256-K stage) units; W, X and residual blocks come from three producer warps.
//  - k_gemm_prefill2 (large M, tensor-bound): 256 tokens x 256 weight rows per pair of
//    CTAs sharing each MMA (cta_group::2).
//  - k_gemm_decode (small M with the activation quantization inside the kernel,
//    mq_gemm_act): a fixed K split per tile, reduced through a thread-block cluster.
// Every kernel is launched with programmatic dependent launch: its prologue overlaps the
// preceding kernel, and it waits for that kernel before touching anything it may write
// (W may be requested earlier when the caller states that it is complete).
#include <algorithm>
#include <atomic>

#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm.cuh"
#include "mosaic_probe.h"
#include "quant.cuh"

namespace mq {

// Device error word (0 = fine, otherwise an mq_status); read and cleared by mq_get_error.
__device__ int g_error = 0;

#ifdef MQ_TIMELINE
// Event times of the first CTAs of the latest small-problem decode launch (mq_timeline_read).
__device__ unsigned long long g_timeline[MQ_TIMELINE_CTAS][MQ_TIMELINE_EVENTS];
#endif
// Records event `ev` of this CTA in a timeline build; nothing otherwise.
__device__ __forceinline__ void tl_event(int ev) {
#ifdef MQ_TIMELINE
    if (blockIdx.x < MQ_TIMELINE_CTAS) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        g_timeline[blockIdx.x][ev] = t;
    }
#else
    (void)ev;
#endif
}

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

// One lane of a converged warp (the same lane every time the full warp calls it).
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred P;\n\t.reg .b32 r;\n\t"
        "elect.sync r|P, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// Bounded wait by a whole warp: all lanes poll, and leave together with lane 0's verdict.
// Role loops (producer, MMA issuer) run converged and let one elected lane issue:
// a loop run by a single lane of an otherwise waiting warp issues far more slowly.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// AND of `v` over the 128 epilogue threads (named barrier 1): every thread leaves with the
// same verdict, so the epilogue warps never split on a wait that ran out for one of them.
__device__ __forceinline__ bool epi_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)(v ? 1 : 0))
        : "memory");
    return r != 0;
}

// mbar_wait_warp with the wall-clock limit given (ns).
__device__ __forceinline__ bool mbar_wait_warp_ns(uint64_t* bar, uint32_t parity, unsigned long long limit) {
    bool ok = mbar_try_wait(bar, parity);
    if (!ok) {
        const unsigned long long t0 = globaltimer();
        while (!(ok = mbar_try_wait(bar, parity)))
            if (globaltimer() - t0 > limit) {
                atomicCAS(&g_error, 0, (int)MQ_ERR_TIMEOUT);
                break;
            }
    }
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

constexpr int kMaxSplits = 16;        // split-K factor bound of the decode plan
constexpr int kMaxClusterSplits = 8;  // splits reduced through a thread-block cluster

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
    static constexpr int kCtrlBytes = 256;  // 3 barriers per stage, accumulator barrier, TMEM address, masks
    // fused activation quantization: per-token partial maxima of every split [8][BN], the
    // token scales [BN], this CTA's partial maxima [BN], the exchange barrier
    static constexpr int kOffFused = kStages * kStageBytes + kCtrlBytes;
    static constexpr int kFusedBytes = (kMaxClusterSplits + 2) * BN * 4 + 16;
    static constexpr int kSmemBytes = kOffFused + kFusedBytes + 1024;
    static constexpr int kThreads = 192;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kSfCol0 = 128;                  // scale columns start after D
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Walks the selected blocks of one block row in increasing block-column order: the
// packed index of the next selected block and the bitmap word being read.
struct RowCursor {
    const uint32_t* words;
    int idx;   // packed index of the first selected block at or after the cursor
    int w;     // index of the bitmap word held in `word`
    uint32_t word;
};

// Cursor at block column kt_begin (a multiple of 4) of block row nt.
__device__ __forceinline__ RowCursor row_cursor(const GemmParams& p, int nt, int kt_begin) {
    const int KW = (p.K / 64 + 31) / 32;
    RowCursor c;
    c.words = p.bitmap + (int64_t)nt * KW;
    c.w = kt_begin >> 5;
    c.word = __ldg(c.words + c.w);
    int idx = __ldg(p.tile_ptr + nt);
    for (int j = 0; j < c.w; ++j) idx += __popc(__ldg(c.words + j));
    const int sh = kt_begin & 31;
    c.idx = idx + __popc(sh ? (c.word & ((1u << sh) - 1u)) : 0u);
    return c;
}

// Presence bits of block columns kt0..kt0+3 (kt0 % 4 == 0, increasing from call to
// call) and the packed index of each present block.
__device__ __forceinline__ uint32_t row_step(RowCursor& c, int kt0, int (&idx)[4]) {
    if ((kt0 >> 5) != c.w) {
        c.w = kt0 >> 5;
        c.word = __ldg(c.words + c.w);
    }
    const uint32_t m = (c.word >> (kt0 & 31)) & 15u;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        idx[kk] = c.idx;
        c.idx += (m >> kk) & 1u;
    }
    return m;
}

__device__ __forceinline__ bool tile_has_mma(const GemmParams& p, int n_tile, int ks_begin, int ks_end) {
    if (ks_end <= ks_begin) return false;
    if (p.mode != 2) return true;
    if (!p.has_resid) return false;
    const int KB = p.K / 64, KW = (KB + 31) / 32;
    for (int h = 0; h < 2; ++h) {
        const uint32_t* row = p.bitmap + (int64_t)(n_tile * 2 + h) * KW;
        for (int kt = ks_begin * 4; kt < ks_end * 4; kt += 4)
            if ((__ldg(row + (kt >> 5)) >> (kt & 31)) & 15u) return true;
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
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);  // W, X and scales landed
    uint64_t* rfull = full + C::kStages;                                                // residual blocks landed
    uint64_t* empty = rfull + C::kStages;                                               // stage consumed
    uint64_t* accf = empty + C::kStages;                                                // accumulator complete
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accf + 1);
    uint32_t* rmask = tmem_holder + 1;  // [kStages]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tile = blockIdx.x, split = blockIdx.y, m_tile = blockIdx.z;
    const int n0 = n_tile * 128, m0 = m_tile * BN;
    const int KS = p.K / 256, KS64 = p.K / 64;
    const int ks_begin = split * p.iters_per_split;
    const int ks_end = min(KS, ks_begin + p.iters_per_split);
    const int n_iters = max(0, ks_end - ks_begin);

    // fused activation quantization (p.x_bf16): warps 2-5 quantize X into the stages
    const bool fused_x = p.x_bf16 != nullptr;
    float* amax_in = reinterpret_cast<float*>(smem + C::kOffFused);  // [kMaxClusterSplits][BN]
    float* g_s = amax_in + kMaxClusterSplits * BN;                      // [BN] token scales
    float* part = g_s + BN;                                             // [BN] this CTA's maxima
    uint64_t* xg_bar = reinterpret_cast<uint64_t*>(part + BN);          // peers' maxima landed
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], fused_x ? 2 : 1);  // + the quantizer warps' arrival
            mbar_init(&rfull[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(xg_bar, fused_x && p.cluster ? p.splits : 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmap_w);
        if (!fused_x) tma_prefetch_desc(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // peers write their activation maxima into this CTA's shared memory: every barrier of
    // the cluster is initialised before any of them starts
    if (fused_x && p.cluster) cluster_sync();

    if (warp == 0) {
        // ---------------------------------------------------- producer (converged warp, one lane issues)
        const uint8_t* xsf_tile = p.x_sf + (int64_t)(m0 / 128) * KS64 * 512;
        const uint8_t* wsf_tile = p.w_sf + (int64_t)n_tile * KS64 * 512;
        // W tile and W scales (the stage's expected bytes are armed here, X's included)
        // (only the residual computed: the dense W tile is not needed)
        const bool dense = p.mode != 2;
        auto issue_w = [&](int it) {
            const int st_i = it % C::kStages, ks = ks_begin + it;
            uint8_t* st = smem + st_i * C::kStageBytes;
            mbar_arrive_expect_tx(&full[st_i], (dense ? 16384 + 2048 : 0) + (fused_x ? 0 : BN * 128 + 2048));
            if (dense) {
                tma_load_2d(st + C::kOffW, &tmap_w, &full[st_i], ks * 128, n0);
                bulk_load(st + C::kOffSFW, wsf_tile + (int64_t)ks * 4 * 512, 2048, &full[st_i]);
            }
        };
        // X tile and X scales
        auto issue_x = [&](int it) {
            if (fused_x) return;  // the quantizer warps write X into the stage
            const int st_i = it % C::kStages, ks = ks_begin + it;
            uint8_t* st = smem + st_i * C::kStageBytes;
            tma_load_2d(st + C::kOffX, &tmap_x, &full[st_i], ks * 128, m0);
            bulk_load(st + C::kOffSFX, xsf_tile + (int64_t)ks * 4 * 512, 2048, &full[st_i]);
        };
        RowCursor cur0, cur1;
        // selected residual blocks of a stage (bit 2*kk + h) and their packed indices
        auto resid_mask = [&](int it, int (&idx0)[4], int (&idx1)[4]) -> uint32_t {
            uint32_t m = 0;
            if (p.has_resid) {
                const int ks = ks_begin + it;
                const uint32_t m0b = row_step(cur0, ks * 4, idx0);
                const uint32_t m1b = row_step(cur1, ks * 4, idx1);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    m |= (((m0b >> kk) & 1u) << (2 * kk)) | (((m1b >> kk) & 1u) << (2 * kk + 1));
            }
            return m;
        };
        auto issue_resid = [&](int it, uint32_t m, const int (&idx0)[4], const int (&idx1)[4]) {
            const int s = it % C::kStages;
            uint8_t* st = smem + s * C::kStageBytes;
            rmask[s] = m;
            mbar_arrive_expect_tx(&rfull[s], __popc(m) * (2048 + 512));
            for (uint32_t mm = m; mm; mm &= mm - 1) {
                const int j = __ffs(mm) - 1, kk = j >> 1, h = j & 1;
                int idx = 0;
#pragma unroll
                for (int a = 0; a < 4; ++a)
                    if (a == kk) idx = h ? idx1[a] : idx0[a];
                idx = min(max(idx, 0), p.nblk - 1);  // a well-formed index is already in range
                bulk_load(st + C::kOffRC + kk * 4096 + h * 2048, p.blk_codes + (int64_t)idx * 2048, 2048,
                          &rfull[s]);
                bulk_load(st + C::kOffRSF + j * 512, p.blk_sf + (int64_t)idx * 512, 512, &rfull[s]);
            }
        };
        const int first = min(C::kStages, n_iters);
        // W and X normally come from earlier kernels of the stream, so they are loaded
        // after the wait for the preceding kernel; a caller that guarantees both were
        // complete before this kernel could start (p.prefetch) lets the first stages load
        // at once, so their base MMAs need not wait for the residual's producer.
        if (!p.prefetch) griddep_wait();
        if (elect_one())
            for (int it = 0; it < first; ++it) {
                issue_w(it);
                issue_x(it);
            }
        __syncwarp();
        if (p.prefetch) griddep_wait();
        // the residual lookups (dependent index loads) run while W and X are in flight;
        // the base MMAs of a stage do not wait for its residual blocks
        if (p.has_resid && n_iters > 0) {
            cur0 = row_cursor(p, n_tile * 2 + 0, ks_begin * 4);
            cur1 = row_cursor(p, n_tile * 2 + 1, ks_begin * 4);
        }
        for (int it = 0; it < first; ++it) {
            int idx0[4] = {0, 0, 0, 0}, idx1[4] = {0, 0, 0, 0};
            const uint32_t m = resid_mask(it, idx0, idx1);
            if (elect_one()) issue_resid(it, m, idx0, idx1);
            __syncwarp();
        }
        int issued = first;
        for (int it = first; it < n_iters; ++it) {
            const int st_i = it % C::kStages;
            if (!mbar_wait_warp(&empty[st_i], ((it / C::kStages) - 1) & 1)) break;
            int idx0[4] = {0, 0, 0, 0}, idx1[4] = {0, 0, 0, 0};
            const uint32_t m = resid_mask(it, idx0, idx1);
            if (elect_one()) {
                issue_w(it);
                issue_x(it);
                issue_resid(it, m, idx0, idx1);
            }
            __syncwarp();
            ++issued;
        }
        // Do not leave while copies into this CTA's shared memory are in flight.
        for (int it = max(0, issued - C::kStages); it < issued; ++it) {
            mbar_wait_warp(&full[it % C::kStages], (it / C::kStages) & 1);
            mbar_wait_warp(&rfull[it % C::kStages], (it / C::kStages) & 1);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer (converged warp, one lane issues)
        constexpr uint32_t idesc = idesc_mxf4nvf4(128, BN);
        uint32_t acc = 0;
        for (int it = 0; it < n_iters; ++it) {
            const int s = it % C::kStages;
            const uint32_t par = (it / C::kStages) & 1;
            if (!mbar_wait_warp(&full[s], par)) break;
            tc_fence_after();
            const uint32_t st = smem_u32(smem + s * C::kStageBytes);
            const uint32_t sfc = tmem + C::kSfCol0 + s * 64;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if (p.mode != 2) tc_cp_sf_chunk(sfc + 4 * kk, smem_desc(st + C::kOffSFW + kk * 512, 0, 128, 0));
                    tc_cp_sf_chunk(sfc + 16 + 4 * kk, smem_desc(st + C::kOffSFX + kk * 512, 0, 128, 0));
                }
                if (p.mode != 2) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_mxf4nvf4(tmem, smem_desc(st + C::kOffW + 32 * kk, 16, 1024, 2),
                                     smem_desc(st + C::kOffX + 32 * kk, 16, 1024, 2), idesc, sfc + 4 * kk,
                                     sfc + 16 + 4 * kk, (acc | kk) != 0);
                    acc = 1;
                }
            }
            __syncwarp();
            acc = __shfl_sync(0xffffffffu, acc, 0);
            if (!mbar_wait_warp(&rfull[s], par)) break;
            tc_fence_after();
            const uint32_t m = p.mode != 1 ? rmask[s] : 0u;
            if (elect_one()) {
                for (uint32_t mm = m; mm; mm &= mm - 1) {
                    const int j = __ffs(mm) - 1, kk = j >> 1;
                    tc_cp_sf_chunk(sfc + 32 + 4 * j, smem_desc(st + C::kOffRSF + j * 512, 0, 128, 0));
                    mma_mxf4nvf4(tmem, smem_desc(st + C::kOffRC + kk * 4096, 128, 256, 0),
                                 smem_desc(st + C::kOffX + 32 * kk, 16, 1024, 2), idesc, sfc + 32 + 4 * j,
                                 sfc + 16 + 4 * kk, acc);
                    acc = 1;
                }
                tc_commit(&empty[s]);
            }
            __syncwarp();
            acc = __shfl_sync(0xffffffffu, acc, 0);
        }
        if (elect_one()) tc_commit(accf);
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (warps 2..5)
        const int q = warp & 3;
        const int nl = 32 * q + lane, n = n0 + nl;
        griddep_wait();  // X, g_x, Y and the workspace follow the previous kernel
        if (fused_x) {
            // ---- activation quantization in the pipeline: per-token maxima over this
            // CTA's K range, exchanged with the cluster's other K splits (or over all of K
            // when the splits do not form a cluster), then every stage's BN x 256 block of
            // X quantized straight into the stage's MMA layout, spread over all 128 threads
            const int tq = threadIdx.x - 64;
            const bool whole_k = p.splits > 1 && !p.cluster;
            const int kb = whole_k ? 0 : ks_begin * 256, kspan = whole_k ? p.K : n_iters * 256;
            {
                // token t = tq / TPT, TPT threads per token striding over its 16-byte vectors
                constexpr int TPT = 128 / BN;
                const int t = tq / TPT, sub = tq % TPT, mm = m0 + t;
                const int nvec = kspan / 8;
                float mx = 0.0f;
                if (mm < p.M) {
                    const uint4* row = reinterpret_cast<const uint4*>(p.x_bf16 + (int64_t)mm * p.K + kb);
                    for (int v0 = sub; v0 < nvec; v0 += TPT * 8) {
                        uint4 x[8];  // eight independent loads in flight
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int v = v0 + TPT * u;
                            x[u] = v < nvec ? __ldg(row + v) : make_uint4(0u, 0u, 0u, 0u);
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                mx = max3(mx, fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)),
                                          fabsf(bf16_bits_to_f32(w[j] >> 16)));
                        }
                    }
                }
#pragma unroll
                for (int o = 1; o < TPT; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (sub == 0) part[t] = mx;
            }
            // the stages' scale rows of tokens >= BN stay zero
            for (int i = tq; i < C::kStages * 128; i += 128)
                reinterpret_cast<uint4*>(smem + (i >> 7) * C::kStageBytes + C::kOffSFX)[i & 127] =
                    make_uint4(0u, 0u, 0u, 0u);
            asm volatile("bar.sync 1, 128;" ::: "memory");
            bool xok = true;
            if (p.cluster) {
                // every split's maxima into every CTA of the cluster, then one arrival each
                const uint32_t S = (uint32_t)p.splits, rank = cluster_ctarank();
                if (tq < BN)
                    for (uint32_t r = 0; r < S; ++r)
                        st_dsmem_f32(mapa_u32(smem_u32(amax_in + rank * BN + tq), r), part[tq]);
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (tq == 0) {
                    fence_acq_rel_cluster();
                    for (uint32_t r = 0; r < S; ++r) mbar_arrive_remote(mapa_u32(smem_u32(xg_bar), r));
                }
                // bounded wait for the S arrivals
                if (!mbar_try_wait_cluster(xg_bar, 0)) {
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try_wait_cluster(xg_bar, 0))
                        if (globaltimer() - t0 > kWaitLimitNs) {
                            atomicCAS(&g_error, 0, (int)MQ_ERR_TIMEOUT);
                            xok = false;
                            break;
                        }
                }
                if (tq < BN) {
                    float mx = 0.0f;
                    for (uint32_t r = 0; r < S; ++r) mx = fmaxf(mx, amax_in[r * BN + tq]);
                    part[tq] = mx;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
            }
            if (tq < BN) {
                const float mx = part[tq];
                g_s[tq] = mx == 0.0f ? 1.0f : __fdiv_rn(mx, 2688.0f);
                if (p.gx_out && n_tile == 0 && split == 0 && m0 + tq < p.M) p.gx_out[m0 + tq] = g_s[tq];
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            // group i = tq + 128 j of a stage: token i / 16, group (i % 16) of its 256 K
            constexpr int GPT = BN * 16 / 128;  // groups per thread and stage
            for (int it = 0; it < n_iters && xok; ++it) {
                const int s = it % C::kStages, ks = ks_begin + it;
                if (it >= C::kStages && !mbar_wait(&empty[s], ((it / C::kStages) - 1) & 1)) { xok = false; break; }
                uint8_t* st = smem + s * C::kStageBytes;
                constexpr int kChunk = GPT < 4 ? GPT : 4;  // groups loaded together
#pragma unroll 1
                for (int j0 = 0; j0 < GPT; j0 += kChunk) {
                float a[kChunk][16];
#pragma unroll
                for (int jj = 0; jj < kChunk; ++jj) {  // the chunk's loads first
                    const int i = tq + 128 * (j0 + jj), t = i >> 4, q16 = i & 15, mm = m0 + t;
                    if (mm < p.M) {
                        load16_bf16(p.x_bf16 + (int64_t)mm * p.K + ks * 256 + q16 * 16, a[jj]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) a[jj][e] = 0.0f;
                    }
                }
#pragma unroll
                for (int jj = 0; jj < kChunk; ++jj) {
                    const int j = j0 + jj;
                    const int i = tq + 128 * j, t = i >> 4, q16 = i & 15, kk = q16 >> 2, gq = q16 & 3;
                    const float g = g_s[t], g6 = __fmul_rn(6.0f, g);
                    float deq[16];
                    uint32_t lo, hi;
                    const uint32_t sfb = nvfp4_group(a[jj], g, g6, lo, hi, deq);
                    // 8 bytes of token row t at byte 8*q16 (128-byte swizzle); the scale in
                    // chunk kk, row t (t < BN <= 128: byte (t%32)*16 + (t/32)*4 + gq)
                    const int c = q16 >> 1;
                    *reinterpret_cast<uint2*>(st + C::kOffX + t * 128 + ((c ^ (t & 7)) << 4) + 8 * (q16 & 1)) =
                        make_uint2(lo, hi);
                    st[C::kOffSFX + kk * 512 + (t & 31) * 16 + (t >> 5) * 4 + gq] = (uint8_t)sfb;
                }
                }
                fence_proxy_async_smem();  // the MMA reads these through the async proxy
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (tq == 0) mbar_arrive(&full[s]);
            }
        }
        const bool waited = mbar_wait(accf, 0);
        tc_fence_after();
        const bool have = waited && tile_has_mma(p, n_tile, ks_begin, ks_end);
        const float gw = __ldg(p.g_w);
        const int Mp = gridDim.z * BN;
        float* red = reinterpret_cast<float*>(smem);  // [BN][128] partial (stages are free now)
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
            float acc[16];
            if (have) {
                tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + c0, acc);
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
            }
            if (p.splits == 1) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int mm = m0 + c0 + j;
                    if (mm < p.M) {
                        const float sc = __fmul_rn(fused_x ? g_s[mm - m0] : __ldg(p.g_x + mm), gw);
                        const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(acc[j], sc));
                        p.Y[(int64_t)mm * p.N + n] = *reinterpret_cast<const uint16_t*>(&y);
                    }
                }
            } else if (p.cluster) {
#pragma unroll
                for (int j = 0; j < 16; ++j) red[(c0 + j) * 128 + nl] = acc[j];
            } else {
                float* part = p.partial + ((int64_t)split * Mp + m0) * p.N + n;
#pragma unroll
                for (int j = 0; j < 16; ++j) __stcg(part + (int64_t)(c0 + j) * p.N, acc[j]);
            }
        }
        tc_fence_before();
        if (p.splits > 1 && !p.cluster) {
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            __shared__ int s_last;
            int* ctr = p.counters + m_tile * gridDim.x + n_tile;
            if (threadIdx.x == 64) s_last = (atomicAdd(ctr, 1) == p.splits - 1);
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (s_last) {
                __threadfence();
                // the last CTA of the tile adds all splits' partials in split order
                const float* base = p.partial + (int64_t)m0 * p.N + n;
                const int64_t sstride = (int64_t)Mp * p.N;
#pragma unroll 1
                for (int c0 = 0; c0 < BN && m0 + c0 < p.M; c0 += 8) {
                    float sum[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) sum[j] = __ldcg(base + (int64_t)(c0 + j) * p.N);
#pragma unroll 4
                    for (int s2 = 1; s2 < p.splits; ++s2) {
                        float v[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) v[j] = __ldcg(base + s2 * sstride + (int64_t)(c0 + j) * p.N);
#pragma unroll
                        for (int j = 0; j < 8; ++j) sum[j] = __fadd_rn(sum[j], v[j]);
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int mm = m0 + c0 + j;
                        if (mm < p.M) {
                            const float sc = __fmul_rn(fused_x ? g_s[mm - m0] : __ldg(p.g_x + mm), gw);
                            const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(sum[j], sc));
                            p.Y[(int64_t)mm * p.N + n] = *reinterpret_cast<const uint16_t*>(&y);
                        }
                    }
                }
                if (threadIdx.x == 64) *ctr = 0;
            }
        }
    }
    griddep_launch();
    if (p.splits > 1 && p.cluster) {
        // every CTA of the cluster holds its partial in shared memory; CTA r adds rows
        // [r*128/S, (r+1)*128/S) of all splits in split order
        __syncwarp();
        cluster_sync();
        if (warp >= 2) {
            const uint32_t S = (uint32_t)p.splits, r = cluster_ctarank();
            const int r0 = (int)(r * 128 / S), r1 = (int)((r + 1) * 128 / S), rows = r1 - r0;
            const float* red = reinterpret_cast<const float*>(smem);
            const float gw = __ldg(p.g_w);
            // kU elements per thread at a time: all their peers' partials are requested
            // before the first add, then added in split order
            constexpr int kU = 4;
            const int total = rows * BN;
            for (int e0 = threadIdx.x - 64; e0 < total; e0 += 128 * kU) {
                float v[kU][kMaxClusterSplits];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int e = min(e0 + 128 * u, total - 1);
                    const int j = e / rows, nl = r0 + e % rows;
#pragma unroll
                    for (uint32_t s2 = 0; s2 < (uint32_t)kMaxClusterSplits; ++s2)
                        if (s2 < S) v[u][s2] = ld_dsmem_f32(red + j * 128 + nl, s2);
                }
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int e = e0 + 128 * u;
                    if (e >= total) break;
                    const int j = e / rows, nl = r0 + e % rows;
                    const int mm = m0 + j;
                    float sum = v[u][0];
#pragma unroll
                    for (uint32_t s2 = 1; s2 < (uint32_t)kMaxClusterSplits; ++s2)
                        if (s2 < S) sum = __fadd_rn(sum, v[u][s2]);
                    if (mm < p.M) {
                        const float sc = __fmul_rn(fused_x ? g_s[mm - m0] : __ldg(p.g_x + mm), gw);
                        const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(sum, sc));
                        p.Y[(int64_t)mm * p.N + n0 + nl] = *reinterpret_cast<const uint16_t*>(&y);
                    }
                }
            }
        }
        __syncwarp();
        cluster_sync();  // peers may still be reading this CTA's partial until here
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Element i of a small per-stage register array (unrolled select, no local memory).
template <int N>
__device__ __forceinline__ int pick(const int (&a)[N], int i) {
    int v = a[0];
#pragma unroll
    for (int j = 1; j < N; ++j)
        if (i == j) v = a[j];
    return v;
}
template <int N>
__device__ __forceinline__ void put(int (&a)[N], int i, int v) {
#pragma unroll
    for (int j = 0; j < N; ++j)
        if (i == j) a[j] = v;
}

// ------------------------------------------------------------------ stream-K decode kernel
// Small M, HBM-bound: every byte of W must stream through the SMs at the full rate of
// the memory. The work is a list of units, (output tile, 256-K stage) pairs, tile-major;
// a grid of one persistent CTA per SM takes equal contiguous ranges of it, so every SM
// streams the same number of W bytes whatever the tile count. A range cuts a tile into
// segments; each segment accumulates in its own tensor-memory buffer (two, alternating,
// so the next segment's MMAs overlap this one's epilogue). A tile held whole by one CTA
// is scaled and stored at once; the segments of a split tile leave fp32 partials in
// per-CTA workspace slots, and the CTA that finishes the tile's last segment (a tile
// counter) adds them in segment order, so the result does not depend on timing.
// Shared memory: a deep ring of stages (W 128 x 256 K, X BN x 256 K, their scale chunks),
// 8 stages for BN = 16 (128 KB of W in flight per SM), and a ring of 16 residual-block
// slots (2048 B codes + 512 B scales each) that a stage's blocks take in order and its
// release frees. A residual block is one M = 128 MMA over its 64 rows and the 2 KB next
// to them in the ring (the other half of the 128-row operand), whose scales are zero.
template <int BN>
struct SKCfg {
    static constexpr int kStages = BN <= 16 ? 8 : BN <= 32 ? 7 : BN <= 64 ? 6 : 5;
    static constexpr int kOffW = 0;                     // 128 rows x 128 B, swizzled
    static constexpr int kOffX = 16384;                 // BN rows x 128 B, swizzled
    static constexpr int kOffSFW = kOffX + BN * 128;    // 4 x 512 B
    static constexpr int kOffSFX = kOffSFW + 2048;      // 4 x 512 B
    static constexpr int kStageBytes = kOffSFX + 2048;
    static constexpr int kRSlots = 16;
    static constexpr int kRSlotBytes = 2560;            // 2048 B codes + 512 B scales
    static constexpr int kOffRing = kStages * kStageBytes;
    // 2 KB after the ring: the last slot's lower-half MMA reads 2 KB past its codes
    static constexpr int kCtrlOff = kOffRing + kRSlots * kRSlotBytes + 2048;
    static constexpr int kMaxSegs = 160;                 // segments of one tile (<= CTAs)
    static constexpr int kCtrlBytes = 512 + 4 * kMaxSegs;
    static constexpr int kSmemBytes = kCtrlOff + kCtrlBytes + 1024;
    static constexpr int kThreads = 256;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kDStride = BN <= 64 ? 64 : 128;        // accumulator buffers
    static constexpr uint32_t kSfCol0 = 2 * kDStride;                  // stage s: 32 columns
    static constexpr uint32_t kRSfCol0 = kSfCol0 + kStages * 32;       // ring slot i: 4 columns
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kRSfCol0 + kRSlots * 4 <= kTmemCols, "tensor memory budget");
};

// CTA holding unit u when `units` are split into `grid` equal contiguous ranges, and the
// first unit of CTA c (units * grid < 2^32, checked on the host: 32-bit arithmetic).
__device__ __forceinline__ uint32_t sk_owner(uint32_t u, uint32_t units, uint32_t grid) {
    return ((u + 1) * grid - 1) / units;
}
__device__ __forceinline__ uint32_t sk_start(uint32_t c, uint32_t units, uint32_t grid) { return c * units / grid; }

// Atomic add with acquire-release semantics at GPU scope: the CTA's partial stores that a
// barrier ordered before it are released with it, and the partials other CTAs released
// before their own increments are acquired.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* ptr, int v) {
    int old;
    asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
    return old;
}

// Does block row pair (n_tile) carry a selected residual block in stages [ks_a, ks_b)?
__device__ __forceinline__ bool resid_in_range(const GemmParams& p, int n_tile, int ks_a, int ks_b) {
    if (!p.has_resid) return false;
    const int KB = p.K / 64, KW = (KB + 31) / 32;
    for (int h = 0; h < 2; ++h) {
        const uint32_t* row = p.bitmap + (int64_t)(n_tile * 2 + h) * KW;
        for (int kt = ks_a * 4; kt < ks_b * 4; kt += 4)
            if ((__ldg(row + (kt >> 5)) >> (kt & 31)) & 15u) return true;
    }
    return false;
}

template <int BN>
__global__ void __launch_bounds__(256, 1)
    k_gemm_streamk(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                   const GemmParams p) {
    using C = SKCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kCtrlOff);  // W, X and scales landed
    uint64_t* rfull = full + C::kStages;                                // residual blocks landed
    uint64_t* empty = rfull + C::kStages;                               // stage and its ring slots consumed
    uint64_t* accf = empty + C::kStages;                                // [2] accumulator complete
    uint64_t* acce = accf + 2;                                          // [2] accumulator read out
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acce + 2);
    uint32_t* rmask = tmem_holder + 1;  // [kStages]: bit 2 * kk + h
    int* s_last = reinterpret_cast<int*>(rmask + C::kStages);
    int* s_slot = s_last + 1;  // [kMaxSegs]: workspace slot of each segment of the tile being added

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KS = p.K / 256, KS64 = p.K / 64;
    const uint32_t U = (uint32_t)p.units, G = gridDim.x;
    const uint32_t u0 = sk_start(blockIdx.x, U, G), u1 = sk_start(blockIdx.x + 1, U, G);
    const int nu = (int)(u1 - u0);
    const bool dense = p.mode != 2;
    const bool resid = p.has_resid && p.mode != 1;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 2);  // the W producer's and the X producer's arrivals
            mbar_init(&rfull[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 4);
        }
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
    const uint32_t sbase = smem_u32(smem);

    // Three producer warps keep the copies of a unit off one another's path: the W stream
    // (the bytes that bound the kernel) never waits for an index lookup or a residual copy.
    if (warp == 0) {
        // ---------------------------------------------------- W producer
        // W may be requested before the wait for the preceding kernel when no running kernel
        // can still write it (the caller's weights-ready guarantee, or the whole-path order)
        if (!(p.prefetch || p.w_ready)) griddep_wait();
        int issued = 0;
        int t = (int)(u0 / (uint32_t)KS), ks = (int)(u0 % (uint32_t)KS);
        for (int i = 0; i < nu; ++i, ks = ks + 1 == KS ? 0 : ks + 1, t += ks == 0) {
            const int s = i % C::kStages;
            if (i >= C::kStages && !mbar_wait_warp_ns(&empty[s], (uint32_t)(((i / C::kStages) - 1) & 1), p.wait_ns)) break;
            // test hook (mq_test_arm_wait_fault): this unit's W is never requested, so the
            // MMA issuer's wait for it runs out with nothing in flight
            if (blockIdx.x == 0 && i == p.skip_unit) continue;
            if (elect_one()) {
                uint8_t* st = smem + s * C::kStageBytes;
                const int n_tile = t / p.tiles_m;
                mbar_arrive_expect_tx(&full[s], dense ? 16384 + 2048 : 0);
                if (dense) {
                    tma_load_2d(st + C::kOffW, &tmap_w, &full[s], ks * 128, n_tile * 128);
                    bulk_load(st + C::kOffSFW, p.w_sf + ((int64_t)n_tile * KS64 + ks * 4) * 512, 2048, &full[s]);
                }
            }
            __syncwarp();
            issued = i + 1;
        }
        // Do not leave while copies into this CTA's shared memory are in flight.
        for (int v = issued > C::kStages ? issued - C::kStages : 0; v < issued; ++v)
            mbar_wait_warp_ns(&full[v % C::kStages], (uint32_t)((v / C::kStages) & 1), p.wait_ns);
    } else if (warp == 2) {
        // ---------------------------------------------------- X producer
        if (!p.prefetch) griddep_wait();
        griddep_launch();
        int issued = 0;
        int t = (int)(u0 / (uint32_t)KS), ks = (int)(u0 % (uint32_t)KS);
        for (int i = 0; i < nu; ++i, ks = ks + 1 == KS ? 0 : ks + 1, t += ks == 0) {
            const int s = i % C::kStages;
            if (i >= C::kStages && !mbar_wait_warp_ns(&empty[s], (uint32_t)(((i / C::kStages) - 1) & 1), p.wait_ns)) break;
            if (elect_one()) {
                uint8_t* st = smem + s * C::kStageBytes;
                const int m_tile = t % p.tiles_m;
                mbar_arrive_expect_tx(&full[s], BN * 128 + 2048);
                tma_load_2d(st + C::kOffX, &tmap_x, &full[s], ks * 128, m_tile * BN);
                bulk_load(st + C::kOffSFX, p.x_sf + ((int64_t)(m_tile * BN / 128) * KS64 + ks * 4) * 512, 2048,
                          &full[s]);
            }
            __syncwarp();
            issued = i + 1;
        }
        for (int v = issued > C::kStages ? issued - C::kStages : 0; v < issued; ++v)
            mbar_wait_warp_ns(&full[v % C::kStages], (uint32_t)((v / C::kStages) & 1), p.wait_ns);
    } else if (warp == 3) {
        // ---------------------------------------------------- residual producer
        // The packed residual may come from the preceding kernel (the whole-path call's
        // pack): only the caller's weights-ready guarantee lets it be read before the wait.
        if (!p.w_ready) griddep_wait();
        int nres = 0;               // units whose residual copies are issued
        int rc = 0, rdone = 0;      // residual blocks issued / known consumed
        int ends[C::kStages] = {};  // rc after the latest unit held by each stage
        RowCursor cur0, cur1;
        int cur_t = -1;
        bool ok = true;
        int t = (int)(u0 / (uint32_t)KS), ks = (int)(u0 % (uint32_t)KS);
        for (int i = 0; i < nu && ok; ++i, ks = ks + 1 == KS ? 0 : ks + 1, t += ks == 0) {
            const int s = i % C::kStages;
            // residual blocks of the unit: both 64-row block rows of the tile, 4 block columns
            uint32_t m = 0;
            int idx0[4] = {0, 0, 0, 0}, idx1[4] = {0, 0, 0, 0};
            if (resid) {
                const int n_tile = t / p.tiles_m;
                if (t != cur_t) {
                    cur0 = row_cursor(p, n_tile * 2 + 0, ks * 4);
                    cur1 = row_cursor(p, n_tile * 2 + 1, ks * 4);
                    cur_t = t;
                }
                const uint32_t m0b = row_step(cur0, ks * 4, idx0);
                const uint32_t m1b = row_step(cur1, ks * 4, idx1);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    m |= (((m0b >> kk) & 1u) << (2 * kk)) | (((m1b >> kk) & 1u) << (2 * kk + 1));
            }
            if (i >= C::kStages) {  // the stage's mask and barrier phase are free again
                if (!mbar_wait_warp_ns(&empty[s], (uint32_t)(((i / C::kStages) - 1) & 1), p.wait_ns)) { ok = false; break; }
                rdone = max(rdone, pick(ends, s));
            }
            const int n = __popc(m);
            // ring slots [rc, rc + n) must be free: wait for younger units until they are
            for (int v = i - C::kStages + 1; rc + n - C::kRSlots > rdone && v < i && ok; ++v) {
                if (v < 0) continue;
                ok = mbar_wait_warp_ns(&empty[v % C::kStages], (uint32_t)((v / C::kStages) & 1), p.wait_ns);
                rdone = max(rdone, pick(ends, v % C::kStages));
            }
            if (!ok) break;
            if (elect_one()) {
                rmask[s] = m;
                mbar_arrive_expect_tx(&rfull[s], n * C::kRSlotBytes);
                int r = rc;
                for (uint32_t mm = m; mm; mm &= mm - 1, ++r) {
                    const int j = __ffs(mm) - 1, kk = j >> 1, h = j & 1;
                    int bi = 0;
#pragma unroll
                    for (int a = 0; a < 4; ++a)
                        if (a == kk) bi = h ? idx1[a] : idx0[a];
                    bi = min(max(bi, 0), p.nblk - 1);  // a well-formed index is already in range
                    const uint32_t slot = sbase + C::kOffRing + (r % C::kRSlots) * C::kRSlotBytes;
                    bulk_load_s(slot, p.blk_codes + (int64_t)bi * 2048, 2048, &rfull[s]);
                    bulk_load_s(slot + 2048, p.blk_sf + (int64_t)bi * 512, 512, &rfull[s]);
                }
            }
            __syncwarp();
            ++nres;
            rc += n;
            put(ends, s, rc);
        }
        for (int v = nres > C::kStages ? nres - C::kStages : 0; v < nres; ++v)
            mbar_wait_warp_ns(&rfull[v % C::kStages], (uint32_t)((v / C::kStages) & 1), p.wait_ns);
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = idesc_mxf4nvf4(128, BN);
        int rc = 0, seg = 0;
        uint32_t acc = 0;
        bool ok = true;
        int ks = (int)(u0 % (uint32_t)KS);
        for (int i = 0; i < nu && ok; ++i, ks = ks + 1 == KS ? 0 : ks + 1) {
            const int s = i % C::kStages;
            const uint32_t par = (uint32_t)((i / C::kStages) & 1);
            const uint32_t d = tmem + (uint32_t)(seg & 1) * C::kDStride;
            if (i == 0 || ks == 0) {  // a segment starts: its accumulator buffer must be free
                if (!mbar_wait_warp_ns(&acce[seg & 1], (uint32_t)(((seg >> 1) & 1) ^ 1), p.wait_ns)) break;
                tc_fence_after();
                acc = 0;
            }
            if (!mbar_wait_warp_ns(&full[s], par, p.wait_ns)) break;
            tc_fence_after();
            const uint32_t st = sbase + s * C::kStageBytes;
            const uint32_t sfc = tmem + C::kSfCol0 + s * 32;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if (dense) tc_cp_sf_chunk(sfc + 4 * kk, smem_desc(st + C::kOffSFW + kk * 512, 0, 128, 0));
                    tc_cp_sf_chunk(sfc + 16 + 4 * kk, smem_desc(st + C::kOffSFX + kk * 512, 0, 128, 0));
                }
                if (dense) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_mxf4nvf4(d, smem_desc(st + C::kOffW + 32 * kk, 16, 1024, 2),
                                     smem_desc(st + C::kOffX + 32 * kk, 16, 1024, 2), idesc, sfc + 4 * kk,
                                     sfc + 16 + 4 * kk, (acc | kk) != 0);
                    acc = 1;
                }
            }
            __syncwarp();
            acc = __shfl_sync(0xffffffffu, acc, 0);
            if (!mbar_wait_warp_ns(&rfull[s], par, p.wait_ns)) break;
            tc_fence_after();
            const uint32_t m = resid ? rmask[s] : 0u;
            if (elect_one()) {
                int r = rc;
                for (uint32_t mm = m; mm; mm &= mm - 1, ++r) {
                    const int j = __ffs(mm) - 1, kk = j >> 1, h = j & 1;
                    const int slot_i = r % C::kRSlots;
                    const uint32_t slot = sbase + C::kOffRing + slot_i * C::kRSlotBytes;
                    const uint32_t rsf = tmem + C::kRSfCol0 + 4 * slot_i;
                    tc_cp_sf_chunk(rsf, smem_desc(slot + 2048, 0, 128, 0));
                    // the block's 64 rows are half h of a 128-row operand; the other half
                    // (2 KB of the ring next to it) has zero scales
                    mma_mxf4nvf4(d, smem_desc(slot - 2048 * h, 128, 256, 0),
                                 smem_desc(st + C::kOffX + 32 * kk, 16, 1024, 2), idesc, rsf, sfc + 16 + 4 * kk,
                                 acc);
                    acc = 1;
                }
                tc_commit(&empty[s]);
            }
            __syncwarp();
            acc = __shfl_sync(0xffffffffu, acc, 0);
            rc += __popc(m);
            if (i == nu - 1 || ks == KS - 1) {  // the segment ends
                if (elect_one()) tc_commit(&accf[seg & 1]);
                __syncwarp();
                ++seg;
            }
        }
    } else {
        // ---------------------------------------------------- epilogue (warps 4..7)
        const int q = warp & 3, row = 32 * q + lane;
        griddep_wait();  // g_x, Y and the workspace follow the previous kernel
        const float gw = __ldg(p.g_w);
        const int tq = threadIdx.x - 128;
        const uint32_t t_first = u0 / (uint32_t)KS, t_last = (u1 - 1) / (uint32_t)KS;
        int seg = 0;
        for (uint32_t t = t_first; t <= t_last; ++t, ++seg) {
            const int n_tile = (int)t / p.tiles_m, m_tile = (int)t % p.tiles_m;
            const uint32_t ta = t * (uint32_t)KS, tb = ta + (uint32_t)KS;  // the tile's units
            const uint32_t sa = max(ta, u0), sb = min(tb, u1);              // this segment's units
            const bool waited = epi_all(mbar_wait_warp_ns(&accf[seg & 1], (uint32_t)((seg >> 1) & 1), p.wait_ns));
            tc_fence_after();
            const bool have = waited && (dense || resid_in_range(p, n_tile, (int)(sa - ta), (int)(sb - ta)));
            float acc[BN];
            tmem_ld_chunks<BN / 16>(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(seg & 1) * C::kDStride,
                                    have ? 0xFFu : 0u, acc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[seg & 1]);  // the buffer is free for segment seg + 2
            if (!waited) break;
            const int m0 = m_tile * BN;
            const int n = n_tile * 128 + row;
            const int c_lo = (int)sk_owner(ta, U, G), c_hi = (int)sk_owner(tb - 1, U, G);
            if (c_lo == c_hi) {
                // the whole tile is this CTA's: scale and store
#pragma unroll
                for (int j = 0; j < BN; ++j) {
                    const int mm = m0 + j;
                    if (mm < p.M) {
                        const float sc = __fmul_rn(__ldg(p.g_x + mm), gw);
                        const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(acc[j], sc));
                        p.Y[(int64_t)mm * p.N + n] = *reinterpret_cast<const uint16_t*>(&y);
                    }
                }
                continue;
            }
            // a split tile: partial into this CTA's slot (first tile of its range: slot 2c,
            // last: 2c + 1), then the tile's last finisher adds every segment in order
            float* mine = p.partial + (size_t)(2 * blockIdx.x + (t == t_first ? 0 : 1)) * (BN * 128);
#pragma unroll
            for (int j = 0; j < BN; ++j) __stcg(mine + j * 128 + row, acc[j]);
            asm volatile("bar.sync 1, 128;" ::: "memory");  // every partial store before the release
            int* ctr = p.counters + t;
            if (tq == 0) *s_last = (atom_add_acq_rel_gpu(ctr, 1) == c_hi - c_lo);
            asm volatile("bar.sync 1, 128;" ::: "memory");  // the acquire before every load below
            if (!*s_last) continue;
            const int nseg = c_hi - c_lo + 1;
            for (int g = tq; g < nseg; g += 128) {
                const uint32_t c = (uint32_t)(c_lo + g);
                s_slot[g] = 2 * (int)c + (sk_start(c, U, G) / (uint32_t)KS == t ? 0 : 1);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            // 16 tokens at a time; the partials of up to 4 segments requested together, then
            // added in segment order
#pragma unroll 1
            for (int j0 = 0; j0 < BN && m0 + j0 < p.M; j0 += 16) {
                float sum[16];
#pragma unroll 1
                for (int g0 = 0; g0 < nseg; g0 += 4) {
                    float v[4][16];
#pragma unroll
                    for (int gg = 0; gg < 4; ++gg) {
                        if (g0 + gg < nseg) {
                            const float* src = p.partial + (size_t)s_slot[g0 + gg] * (BN * 128) + j0 * 128 + row;
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) v[gg][jj] = __ldcg(src + jj * 128);
                        }
                    }
#pragma unroll
                    for (int gg = 0; gg < 4; ++gg) {
                        if (g0 + gg < nseg) {
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) sum[jj] = g0 + gg ? __fadd_rn(sum[jj], v[gg][jj]) : v[gg][jj];
                        }
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int mm = m0 + j0 + jj;
                    if (mm < p.M) {
                        const float sc = __fmul_rn(__ldg(p.g_x + mm), gw);
                        const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(sum[jj], sc));
                        p.Y[(int64_t)mm * p.N + n] = *reinterpret_cast<const uint16_t*>(&y);
                    }
                }
            }
            if (tq == 0) *ctr = 0;
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Which 64-column slices of a tile's accumulator receive an MMA (bit h: weight rows
// 64h..64h+63)? All of them unless only the residual is computed, in which case a slice
// is written only if its block row has selected blocks.
__device__ __forceinline__ uint32_t prefill_tile_slices(const GemmParams& p, int n_tile) {
    if (p.mode != 2) return 0xFu;
    if (!p.has_resid) return 0u;
    uint32_t m = 0;
    for (int h = 0; h < 4; ++h)
        if (__ldg(p.tile_ptr + n_tile * 4 + h + 1) > __ldg(p.tile_ptr + n_tile * 4 + h)) m |= 1u << h;
    return m;
}

// ------------------------------------------------------------------ small decode kernel
// Decode problems too small to keep every SM streaming for long (LLaMA3-8B q_proj at 16
// tokens: 10.5 MB) are bound by fixed latencies: the wait for the preceding kernel, the
// first data's latency, the reduce-sum. This variant splits each 128-row tile's K range
// evenly among the S CTAs of one thread-block cluster (S <= 8, tiles x S <= SMs) and adds
// the S fp32 partials through the cluster's shared memory, in split order. A CTA is small
// enough for two to share an SM (3-4 stages, an 8-slot residual ring, 256 tensor-memory
// columns), so the next call's CTAs are already resident while this call finishes and,
// when the caller states that the weight is ready (MQ_GEMM_WEIGHTS_READY), stream their W
// meanwhile. Warp 0 issues every copy (W, X, residual blocks), warp 1 the MMAs, warps 2-5
// the epilogue.
template <int BN>
struct SmallCfg {
    static constexpr int kStages = BN <= 16 ? 4 : 3;
    static constexpr int kOffW = 0;                     // 128 rows x 128 B, swizzled
    static constexpr int kOffX = 16384;                 // BN rows x 128 B, swizzled
    static constexpr int kOffSFW = kOffX + BN * 128;    // 4 x 512 B
    static constexpr int kOffSFX = kOffSFW + 2048;      // 4 x 512 B
    static constexpr int kStageBytes = kOffSFX + 2048;
    static constexpr int kRSlots = 8;
    static constexpr int kRSlotBytes = 2560;
    static constexpr int kOffRing = kStages * kStageBytes;
    static constexpr int kCtrlOff = kOffRing + kRSlots * kRSlotBytes + 2048;  // 2 KB after the ring
    static constexpr int kCtrlBytes = 256;
    static constexpr int kSmemBytes = kCtrlOff + kCtrlBytes + 1024;
    static constexpr int kThreads = 192;
    static constexpr uint32_t kTmemCols = 256;
    static constexpr uint32_t kSfCol0 = 32;                          // after D (BN <= 32 columns)
    static constexpr uint32_t kRSfCol0 = kSfCol0 + kStages * 32;
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
    static_assert(kSmemBytes <= 113 * 1024, "two CTAs per SM");
    static_assert(kRSfCol0 + kRSlots * 4 <= kTmemCols, "tensor memory budget");
    static_assert(kStages * kStageBytes >= BN * 128 * 4, "the partial fits in the stage area");
};

template <int BN>
__global__ void __launch_bounds__(192, 2)
    k_gemm_small(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                 const GemmParams p) {
    using C = SmallCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kCtrlOff);  // W, X and scales landed
    uint64_t* rfull = full + C::kStages;                                // residual blocks landed
    uint64_t* empty = rfull + C::kStages;                               // stage and its ring slots consumed
    uint64_t* accf = empty + C::kStages;                                // accumulator complete
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accf + 1);
    uint32_t* rmask = tmem_holder + 1;  // [kStages]: bit 2 * kk + h

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.splits;
    const int tile = blockIdx.x / S, split = blockIdx.x % S;  // split = rank in the (S, 1, 1) cluster
    const int n_tile = tile / p.tiles_m, m_tile = tile % p.tiles_m;
    const int KS = p.K / 256, KS64 = p.K / 64;
    const int ks0 = split * KS / S, nu = (split + 1) * KS / S - ks0;
    const bool dense = p.mode != 2;
    const bool resid = p.has_resid && p.mode != 1;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&rfull[s], 1);
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
    const uint32_t sbase = smem_u32(smem);
    if (threadIdx.x == 0) tl_event(0);

    if (warp == 0) {
        // ---------------------------------------------------- producer: W, X, residual blocks
        auto issue_w = [&](int i) {
            // test hook (mq_test_arm_wait_fault): this unit's W is never requested, so the
            // MMA issuer's wait for it runs out with nothing in flight
            if (blockIdx.x == 0 && i == p.skip_unit) return;
            const int s = i % C::kStages, ks = ks0 + i;
            uint8_t* st = smem + s * C::kStageBytes;
            mbar_arrive_expect_tx(&full[s], (dense ? 16384 + 2048 : 0) + BN * 128 + 2048);
            if (dense) {
                tma_load_2d(st + C::kOffW, &tmap_w, &full[s], ks * 128, n_tile * 128);
                bulk_load(st + C::kOffSFW, p.w_sf + ((int64_t)n_tile * KS64 + ks * 4) * 512, 2048, &full[s]);
            }
        };
        auto issue_x = [&](int i) {
            const int s = i % C::kStages, ks = ks0 + i;
            uint8_t* st = smem + s * C::kStageBytes;
            tma_load_2d(st + C::kOffX, &tmap_x, &full[s], ks * 128, m_tile * BN);
            bulk_load(st + C::kOffSFX, p.x_sf + ((int64_t)(m_tile * BN / 128) * KS64 + ks * 4) * 512, 2048,
                      &full[s]);
        };
        const int first = nu < C::kStages ? nu : C::kStages;
        const bool w_early = p.prefetch || p.w_ready;
        if (w_early && elect_one()) {
            for (int i = 0; i < first; ++i) issue_w(i);
            tl_event(1);
        }
        __syncwarp();
        if (!p.w_ready) {
            griddep_wait();  // the packed residual may come from the preceding kernel
            if (lane == 0) tl_event(2);
        }
        RowCursor cur0, cur1;
        if (resid) {
            cur0 = row_cursor(p, n_tile * 2 + 0, ks0 * 4);
            cur1 = row_cursor(p, n_tile * 2 + 1, ks0 * 4);
        }
        int rc = 0, rdone = 0, nres = 0, nbase = 0;
        int ends[C::kStages] = {};
        bool waited = !p.w_ready, ok = true;
        for (int i = 0; i < nu && ok; ++i) {
            const int s = i % C::kStages;
            if (i >= C::kStages) {
                if (!mbar_wait_warp_ns(&empty[s], (uint32_t)(((i / C::kStages) - 1) & 1), p.wait_ns)) break;
                rdone = max(rdone, pick(ends, s));
            }
            // W (unless requested before the wait) and X: X only after the wait
            if (i >= first || !w_early) {
                if (!waited && !p.prefetch) { griddep_wait(); waited = true; }
                if (elect_one()) {
                    issue_w(i);
                    if (i == 0) tl_event(1);
                }
                __syncwarp();
            }
            if (!waited && !p.prefetch) {
                griddep_wait();
                waited = true;
                if (lane == 0) tl_event(2);
            }
            if (elect_one()) {
                issue_x(i);
                if (i == 0) tl_event(3);
            }
            __syncwarp();
            nbase = i + 1;
            uint32_t m = 0;
            int idx0[4] = {0, 0, 0, 0}, idx1[4] = {0, 0, 0, 0};
            if (resid) {
                const uint32_t m0b = row_step(cur0, (ks0 + i) * 4, idx0);
                const uint32_t m1b = row_step(cur1, (ks0 + i) * 4, idx1);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    m |= (((m0b >> kk) & 1u) << (2 * kk)) | (((m1b >> kk) & 1u) << (2 * kk + 1));
            }
            const int n = __popc(m);
            for (int v = i - C::kStages + 1; rc + n - C::kRSlots > rdone && v < i && ok; ++v) {
                if (v < 0) continue;
                ok = mbar_wait_warp_ns(&empty[v % C::kStages], (uint32_t)((v / C::kStages) & 1), p.wait_ns);
                rdone = max(rdone, pick(ends, v % C::kStages));
            }
            if (!ok) break;
            if (elect_one()) {
                rmask[s] = m;
                mbar_arrive_expect_tx(&rfull[s], n * C::kRSlotBytes);
                int r = rc;
                for (uint32_t mm = m; mm; mm &= mm - 1, ++r) {
                    const int j = __ffs(mm) - 1, kk = j >> 1, h = j & 1;
                    int bi = 0;
#pragma unroll
                    for (int a = 0; a < 4; ++a)
                        if (a == kk) bi = h ? idx1[a] : idx0[a];
                    bi = min(max(bi, 0), p.nblk - 1);  // a well-formed index is already in range
                    const uint32_t slot = sbase + C::kOffRing + (r % C::kRSlots) * C::kRSlotBytes;
                    bulk_load_s(slot, p.blk_codes + (int64_t)bi * 2048, 2048, &rfull[s]);
                    bulk_load_s(slot + 2048, p.blk_sf + (int64_t)bi * 512, 512, &rfull[s]);
                }
            }
            __syncwarp();
            nres = i + 1;
            rc += n;
            put(ends, s, rc);
        }
        if (!waited && !p.prefetch) griddep_wait();
        griddep_launch();
        // Do not leave while copies into this CTA's shared memory are in flight.
        const int nw = w_early ? (nbase > first ? nbase : first) : nbase;
        for (int v = nw > C::kStages ? nw - C::kStages : 0; v < nw; ++v)
            mbar_wait_warp_ns(&full[v % C::kStages], (uint32_t)((v / C::kStages) & 1), p.wait_ns);
        for (int v = nres > C::kStages ? nres - C::kStages : 0; v < nres; ++v)
            mbar_wait_warp_ns(&rfull[v % C::kStages], (uint32_t)((v / C::kStages) & 1), p.wait_ns);
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = idesc_mxf4nvf4(128, BN);
        int rc = 0;
        uint32_t acc = 0;
        for (int i = 0; i < nu; ++i) {
            const int s = i % C::kStages;
            const uint32_t par = (uint32_t)((i / C::kStages) & 1);
            if (!mbar_wait_warp_ns(&full[s], par, p.wait_ns)) break;
            if (i == 0 && lane == 0) tl_event(4);
            tc_fence_after();
            const uint32_t st = sbase + s * C::kStageBytes;
            const uint32_t sfc = tmem + C::kSfCol0 + s * 32;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if (dense) tc_cp_sf_chunk(sfc + 4 * kk, smem_desc(st + C::kOffSFW + kk * 512, 0, 128, 0));
                    tc_cp_sf_chunk(sfc + 16 + 4 * kk, smem_desc(st + C::kOffSFX + kk * 512, 0, 128, 0));
                }
                if (dense) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_mxf4nvf4(tmem, smem_desc(st + C::kOffW + 32 * kk, 16, 1024, 2),
                                     smem_desc(st + C::kOffX + 32 * kk, 16, 1024, 2), idesc, sfc + 4 * kk,
                                     sfc + 16 + 4 * kk, (acc | kk) != 0);
                    acc = 1;
                }
            }
            __syncwarp();
            acc = __shfl_sync(0xffffffffu, acc, 0);
            if (!mbar_wait_warp_ns(&rfull[s], par, p.wait_ns)) break;
            tc_fence_after();
            const uint32_t m = resid ? rmask[s] : 0u;
            if (elect_one()) {
                int r = rc;
                for (uint32_t mm = m; mm; mm &= mm - 1, ++r) {
                    const int j = __ffs(mm) - 1, kk = j >> 1, h = j & 1;
                    const int slot_i = r % C::kRSlots;
                    const uint32_t slot = sbase + C::kOffRing + slot_i * C::kRSlotBytes;
                    const uint32_t rsf = tmem + C::kRSfCol0 + 4 * slot_i;
                    tc_cp_sf_chunk(rsf, smem_desc(slot + 2048, 0, 128, 0));
                    mma_mxf4nvf4(tmem, smem_desc(slot - 2048 * h, 128, 256, 0),
                                 smem_desc(st + C::kOffX + 32 * kk, 16, 1024, 2), idesc, rsf, sfc + 16 + 4 * kk, acc);
                    acc = 1;
                }
                tc_commit(&empty[s]);
            }
            __syncwarp();
            acc = __shfl_sync(0xffffffffu, acc, 0);
            rc += __popc(m);
        }
        if (elect_one()) {
            tc_commit(accf);
            tl_event(5);
        }
        __syncwarp();
    }
    // ---------------------------------------------------- epilogue (warps 2..5)
    // the accumulator of this CTA's K range; with S > 1 it goes to shared memory (the stage
    // area: every MMA has completed) and the cluster adds the S partials in split order
    float* part = reinterpret_cast<float*>(smem);  // [BN][128]
    const int q = warp & 3, row = 32 * q + lane;
    bool ok = true;
    if (warp >= 2) {
        griddep_wait();  // g_x and Y follow the preceding kernel
        ok = epi_all(mbar_wait_warp_ns(accf, 0, p.wait_ns));
        if (threadIdx.x == 64) tl_event(6);
        tc_fence_after();
        const bool have = ok && (dense || resid_in_range(p, n_tile, ks0, ks0 + nu));
        float acc[BN];
        tmem_ld_chunks<BN / 16>(tmem + ((uint32_t)(32 * q) << 16), have ? 0xFFu : 0u, acc);
        tc_fence_before();
        const float gw = __ldg(p.g_w);
        const int m0 = m_tile * BN, n = n_tile * 128 + row;
        if (S == 1) {
#pragma unroll
            for (int j = 0; j < BN; ++j) {
                const int mm = m0 + j;
                if (ok && mm < p.M) {
                    const float sc = __fmul_rn(__ldg(p.g_x + mm), gw);
                    const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(acc[j], sc));
                    p.Y[(int64_t)mm * p.N + n] = *reinterpret_cast<const uint16_t*>(&y);
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < BN; ++j) part[j * 128 + row] = acc[j];
        }
    }
    if (S > 1) {
        // every CTA of the cluster holds its partial; CTA r adds rows [r*128/S, (r+1)*128/S)
        __syncwarp();
        cluster_sync();
        if (threadIdx.x == 64) tl_event(7);
        if (warp >= 2) {
            // rows [r0, r1) of every token, four rows (a 16-byte run of each CTA's partial)
            // per work item: one 16-byte DSMEM load per split instead of four scalar ones
            const int r0 = split * 128 / S, r1 = (split + 1) * 128 / S;
            const int q0 = r0 >> 2, q1 = (r1 + 3) >> 2;  // the 4-row runs touching [r0, r1)
            const float gw = __ldg(p.g_w);
            const int m0 = m_tile * BN;
            const int total = (q1 - q0) * BN;
            for (int e = threadIdx.x - 64; e < total; e += 128) {
                const int j = e / (q1 - q0), nq = 4 * (q0 + e % (q1 - q0));
                float4 v[8];
#pragma unroll
                for (int s2 = 0; s2 < 8; ++s2)
                    if (s2 < S) v[s2] = ld_dsmem_f32x4(part + j * 128 + nq, (uint32_t)s2);
                float4 sum = v[0];
#pragma unroll
                for (int s2 = 1; s2 < 8; ++s2)
                    if (s2 < S) {
                        sum.x = __fadd_rn(sum.x, v[s2].x);
                        sum.y = __fadd_rn(sum.y, v[s2].y);
                        sum.z = __fadd_rn(sum.z, v[s2].z);
                        sum.w = __fadd_rn(sum.w, v[s2].w);
                    }
                const int mm = m0 + j;
                if (ok && mm < p.M) {
                    const float sc = __fmul_rn(__ldg(p.g_x + mm), gw);
                    const float r4[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int nl = nq + u;
                        if (nl < r0 || nl >= r1) continue;  // a run that straddles the range
                        const __nv_bfloat16 y = __float2bfloat16_rn(__fmul_rn(r4[u], sc));
                        p.Y[(int64_t)mm * p.N + n_tile * 128 + nl] = *reinterpret_cast<const uint16_t*>(&y);
                    }
                }
            }
        }
        if (threadIdx.x == 64) tl_event(8);
        __syncwarp();
        cluster_sync();  // peers may still be reading this CTA's partial until here
        if (threadIdx.x == 64) tl_event(9);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ prefill kernel, CTA pairs
// Large M with the tensor cores of two SMs on one 256 x 256 tile (tokens x weight rows):
// a cluster of two CTAs shares every MMA (tcgen05 cta_group::2, issued by the even CTA).
// Each CTA stages its own 128 tokens of X, its own half (128 rows) of the 256 weight rows
// and the scales, so an SM brings in 32 KB of operands per 256-K stage where a CTA that
// computed a 128 x 256 tile alone would bring in 48 KB: the per-SM ingest that bounds the
// single-CTA kernel drops by a third. Both CTAs' copies complete on the even CTA's stage
// barrier; the MMA's completion is signalled to both CTAs' barriers at once. A selected
// residual block is one M = 256, N = 64 MMA into its 64-column slice of the accumulator,
// its 64 weight rows split 32 + 32 between the pair. Each CTA's epilogue drains its own
// 128 accumulator rows. In the even CTA a scale warp copies each stage's scale chunks into
// tensor memory and signals a barrier, so the MMA-issuing thread issues MMAs only (a stage
// has 12 scale copies for 4 MMAs: issued from one thread they took about as long as the
// MMAs run).
struct Prefill2Cfg {
    static constexpr int kStages = 4;
    static constexpr int kOffX = 0;                      // 128 rows x 128 B, swizzled
    static constexpr int kOffW = 16384;                  // 128 rows x 128 B, swizzled
    static constexpr int kOffSFX = 32768;                // 4 x 512 B
    static constexpr int kOffSFW = kOffSFX + 2048;       // 2 row tiles x 4 x 512 B
    static constexpr int kStageBytes = kOffSFW + 4096;   // 38912
    static constexpr int kRSlots = 16;
    static constexpr int kRSlotBytes = 1536;             // 1024 B (32 rows) of codes + 512 B scales
    static constexpr int kOffRing = kStages * kStageBytes;
    static constexpr int kCtrlOff = kOffRing + kRSlots * kRSlotBytes;
    static constexpr int kCtrlBytes = 512;
    static constexpr int kSmemBytes = kCtrlOff + kCtrlBytes + 1024;
    static constexpr int kThreads = 320;  // 0 producer, 1 MMA (even CTA), 2-9 epilogue
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kSfCol0 = 256;                  // after the 256-column accumulator
    static constexpr int kSfStageCols = 48;              // X: 4 x 4, W: 4 x 8
    static constexpr int kRSfCol0 = kSfCol0 + kStages * kSfStageCols;
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kRSfCol0 + kRSlots * 4 <= 512, "tensor memory budget");
};

// AND of `v` over the 256 epilogue threads of the pair kernel (named barrier 1).
__device__ __forceinline__ bool epi_all256(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 256, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)(v ? 1 : 0))
        : "memory");
    return r != 0;
}

// try_wait on a barrier whose completing arrivals come from both CTAs of the pair.
__device__ __forceinline__ bool mbar_wait_warp_cluster(uint64_t* bar, uint32_t parity) {
    bool ok = mbar_try_wait_cluster(bar, parity);
    if (!ok) {
        const unsigned long long t0 = globaltimer();
        while (!(ok = mbar_try_wait_cluster(bar, parity)))
            if (globaltimer() - t0 > kWaitLimitNs) {
                atomicCAS(&g_error, 0, (int)MQ_ERR_TIMEOUT);
                break;
            }
    }
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__global__ void __launch_bounds__(Prefill2Cfg::kThreads, 1)
    k_gemm_prefill2(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                    const __grid_constant__ CUtensorMap tmap_wsf, const __grid_constant__ CUtensorMap tmap_xsf,
                    const __grid_constant__ CUtensorMap tmap_rc, const __grid_constant__ CUtensorMap tmap_rsf,
                    const GemmParams p) {
    using C = Prefill2Cfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kCtrlOff);  // (even CTA) both CTAs' copies landed
    uint64_t* empty = full + C::kStages;                                // stage and its ring slots consumed
    uint64_t* accf = empty + C::kStages;                                // accumulator complete
    uint64_t* acce = accf + 1;                                          // (even CTA) both epilogues read it
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acce + 1);
    uint32_t* rmask = tmem_holder + 1;  // [kStages] (even CTA): bit 4 * kk + h

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int KS = p.K / 256, KS64 = p.K / 64;
    const int tiles_m = (p.M + 255) / 256, tiles_n = p.N / 256;
    const int ntiles = tiles_m * tiles_n;
    const bool dense = p.mode != 2;
    const bool resid = p.has_resid && p.mode != 1;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // The even CTA's producer arrives with the bytes of both CTAs. A stage carrying
            // copies from both CTAs cannot complete before the odd CTA issued it; with only
            // the residual computed, a stage may carry none, so the odd CTA's producer also
            // arrives: either way its view of its empty barrier never falls two phases behind.
            mbar_init(&full[s], p.mode == 2 ? 2 : 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, 16);  // 8 epilogue warps of each CTA
        mbar_fence_init();
        tma_prefetch_desc(&tmap_w);
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_wsf);
        tma_prefetch_desc(&tmap_xsf);
        if (resid) {
            tma_prefetch_desc(&tmap_rc);
            tma_prefetch_desc(&tmap_rsf);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    // both CTAs' barriers initialised and tensor memory allocated before either goes on
    __syncwarp();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ---------------------------------------------------- producer (both CTAs)
        griddep_wait();
        griddep_launch();
        int sc = 0, rc = 0;  // stages and residual blocks issued so far
        int rdone = 0;       // residual blocks known consumed
        int ends[C::kStages] = {};
        bool ok = true;
        for (int t = pair; t < ntiles && ok; t += npairs) {
            const int m_tile = t % tiles_m, n_tile = t / tiles_m;
            RowCursor cur[4];
            if (resid)
#pragma unroll
                for (int h = 0; h < 4; ++h) cur[h] = row_cursor(p, n_tile * 4 + h, 0);
            for (int ks = 0; ks < KS && ok; ++ks, ++sc) {
                const int s = sc % C::kStages;
                if (sc >= C::kStages) {
                    if (!mbar_wait_warp(&empty[s], ((sc / C::kStages) & 1) ^ 1)) { ok = false; break; }
                    rdone = max(rdone, pick(ends, s));
                }
                uint32_t m = 0;
                int idx[4][4];
                if (resid)
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const uint32_t mb = row_step(cur[h], ks * 4, idx[h]);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) m |= ((mb >> kk) & 1u) << (4 * kk + h);
                    }
                const int n = __popc(m);
                // ring slots of blocks released with earlier stages
                for (int u = sc - C::kStages + 1; rc + n - C::kRSlots > rdone && u < sc && ok; ++u) {
                    if (u < 0) continue;
                    ok = mbar_wait_warp(&empty[u % C::kStages], (u / C::kStages) & 1);
                    rdone = max(rdone, pick(ends, u % C::kStages));
                }
                if (!ok) break;
                if (elect_one()) {
                    const bool xneed = dense || n > 0;
                    const uint32_t bar = mapa_u32(smem_u32(&full[s]), 0);
                    uint8_t* st = smem + s * C::kStageBytes;
                    if (leader) {
                        rmask[s] = m;
                        mbar_arrive_expect_tx(&full[s], 2u * ((dense ? 16384 + 4096 : 0) + (xneed ? 16384 + 2048 : 0) +
                                                              n * C::kRSlotBytes));
                    }
                    if (xneed) {
                        tma_load_2d_pair(st + C::kOffX, &tmap_x, bar, ks * 128, m_tile * 256 + 128 * (int)rank);
                        tma_load_2d_pair(st + C::kOffSFX, &tmap_xsf, bar, 0, (m_tile * 2 + (int)rank) * KS64 + ks * 4);
                    }
                    if (dense) {
                        tma_load_2d_pair(st + C::kOffW, &tmap_w, bar, ks * 128, n_tile * 256 + 128 * (int)rank);
                        tma_load_2d_pair(st + C::kOffSFW, &tmap_wsf, bar, 0, (n_tile * 2) * KS64 + ks * 4);
                        tma_load_2d_pair(st + C::kOffSFW + 2048, &tmap_wsf, bar, 0, (n_tile * 2 + 1) * KS64 + ks * 4);
                    }
                    // residual blocks in (kk, h) order into consecutive ring slots: this
                    // CTA's 32 rows of each block, and the block's whole scale chunk
                    int r = rc;
                    for (uint32_t mm = m; mm; mm &= mm - 1, ++r) {
                        const int j = __ffs(mm) - 1, kk = j >> 2, h = j & 3;
                        int bi = 0;
#pragma unroll
                        for (int a = 0; a < 4; ++a)
#pragma unroll
                            for (int b = 0; b < 4; ++b)
                                if (a == h && b == kk) bi = idx[a][b];
                        bi = min(max(bi, 0), p.nblk - 1);  // a well-formed index is already in range
                        uint8_t* slot = smem + C::kOffRing + (r % C::kRSlots) * C::kRSlotBytes;
                        tma_load_2d_pair(slot, &tmap_rc, bar, 0, 2 * bi + (int)rank);
                        tma_load_2d_pair(slot + 1024, &tmap_rsf, bar, 0, bi);
                    }
                    if (!leader && p.mode == 2) mbar_arrive_remote(bar);  // this CTA's copies are issued
                }
                __syncwarp();
                rc += n;
                put(ends, s, rc);
            }
        }
        // Do not leave while copies are in flight: the even CTA's barrier counts both CTAs'
        // bytes (the odd CTA waits for the even one at the closing cluster barrier).
        if (leader)
            for (int u = max(0, sc - C::kStages); u < sc; ++u)
                mbar_wait_warp_cluster(&full[u % C::kStages], (u / C::kStages) & 1);
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer (even CTA)
        if (leader) {
            constexpr uint32_t idesc_d = idesc_mxf4nvf4(256, 256);
            constexpr uint32_t idesc_r = idesc_mxf4nvf4(256, 64);
            // stage 0's descriptors; a stage or K step moves the start address field only
            const uint64_t xd0 = smem_desc(sbase + C::kOffX, 16, 1024, 2);
            const uint64_t wd0 = smem_desc(sbase + C::kOffW, 16, 1024, 2);
            const uint64_t rd0 = smem_desc(sbase + C::kOffRing, 128, 256, 0);
            const uint64_t sd0 = smem_desc(sbase, 0, 128, 0);
            int sc = 0, rc = 0, tc = 0;
            bool ok = true;
            for (int t = pair; t < ntiles && ok; t += npairs, ++tc) {
                uint32_t acc4 = 0;  // bit h: slice h already holds a partial sum
                for (int ks = 0; ks < KS; ++ks, ++sc) {
                    const int s = sc % C::kStages;
                    const uint32_t par = (sc / C::kStages) & 1;
                    if (!mbar_wait_warp_cluster(&full[s], par)) { ok = false; break; }  // rmask[s] is written
                    const uint32_t m = resid ? rmask[s] : 0u;
                    tc_fence_after();
                    const uint64_t so = (uint64_t)((s * C::kStageBytes) >> 4);
                    const uint32_t sfc = tmem + C::kSfCol0 + s * C::kSfStageCols;
                    if (elect_one()) {
                        // the stage's scales into tensor memory, issued ahead of the MMAs that
                        // read them from the same thread (the pipe runs them in order); a
                        // stage's columns, and a ring slot's, are rewritten only after the
                        // MMAs that read them completed (the stage was released first)
                        const uint64_t st = sd0 + so;
                        if (dense || m) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                tc_cp_sf_chunk_pair(sfc + 4 * kk, st + ((C::kOffSFX + kk * 512) >> 4));
                        }
                        if (dense) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                tc_cp_sf_chunk_pair(sfc + 16 + 8 * kk, st + ((C::kOffSFW + kk * 512) >> 4));
                                tc_cp_sf_chunk_pair(sfc + 16 + 8 * kk + 4, st + ((C::kOffSFW + 2048 + kk * 512) >> 4));
                            }
                        }
                        {
                            int r = rc;
                            for (uint32_t mm = m; mm; mm &= mm - 1, ++r) {
                                const int slot_i = r % C::kRSlots;
                                tc_cp_sf_chunk_pair(tmem + C::kRSfCol0 + 4 * slot_i,
                                                    sd0 + (uint64_t)((C::kOffRing + slot_i * C::kRSlotBytes + 1024) >> 4));
                            }
                        }
                    }
                    if (ks == 0) {
                        // A tile's first scale copies go into the pipe before the wait for
                        // both epilogues to have read the previous tile's accumulator: they
                        // write scale columns only, and run while the accumulator drains.
                        __syncwarp();
                        if (!mbar_wait_warp_cluster(acce, (tc & 1) ^ 1)) { ok = false; break; }
                        tc_fence_after();
                    }
                    if (elect_one()) {
                        if (dense) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_mxf4nvf4_pair(tmem, xd0 + so + 2 * kk, wd0 + so + 2 * kk, idesc_d, sfc + 4 * kk,
                                                  sfc + 16 + 8 * kk, (acc4 | kk) != 0);
                            acc4 = 0xFu;
                        }
                        int r = rc;
                        for (uint32_t mm = m; mm; mm &= mm - 1, ++r) {
                            const int j = __ffs(mm) - 1, kk = j >> 2, h = j & 3;
                            const int slot_i = r % C::kRSlots;
                            mma_mxf4nvf4_pair(tmem + 64 * h, xd0 + so + 2 * kk,
                                              rd0 + (uint64_t)((slot_i * C::kRSlotBytes) >> 4), idesc_r, sfc + 4 * kk,
                                              tmem + C::kRSfCol0 + 4 * slot_i + 2 * (h & 1), (acc4 >> h) & 1u);
                            acc4 |= 1u << h;
                        }
                        // both CTAs' stage (and ring slots) are free once these MMAs complete
                        tc_commit_pair_mc(&empty[s], 0x3);
                    }
                    __syncwarp();
                    acc4 = __shfl_sync(0xffffffffu, acc4, 0);
                    rc += __popc(m);
                }
                if (ok && elect_one()) tc_commit_pair_mc(accf, 0x3);
                __syncwarp();
            }
        }
    } else {
        // ---------------------------------------------------- epilogue (warps 2..9, both CTAs)
        const int q = warp & 3, half = (warp - 2) >> 2;
        griddep_wait();  // g_x and Y follow the previous kernel
        const float gw = __ldg(p.g_w);
        const uint32_t acce_even = mapa_u32(smem_u32(acce), 0);
        int tc = 0;
        for (int t = pair; t < ntiles; t += npairs, ++tc) {
            const int m_tile = t % tiles_m, n_tile = t / tiles_m;
            // this thread's row and its scale, loaded before the accumulator is waited for
            const int mm = m_tile * 256 + 128 * (int)rank + 32 * q + lane;
            const float sc = mm < p.M ? __fmul_rn(__ldg(p.g_x + mm), gw) : 0.0f;
            const bool waited = epi_all256(mbar_wait_warp(accf, tc & 1));
            tc_fence_after();
            const uint32_t slices = waited ? prefill_tile_slices(p, n_tile) : 0u;
            // this thread's row: 128 columns (two 64-column slices), all eight loads in flight
            // together; the accumulator is released before the scaling and the stores
            float v[128];
            tmem_ld_chunks<8>(tmem + ((uint32_t)(32 * q) << 16) + 128 * half,
                              ((slices >> (2 * half)) & 1u ? 0x0Fu : 0u) | ((slices >> (2 * half + 1)) & 1u ? 0xF0u : 0u),
                              v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(acce_even);  // this CTA's rows are read
            if (!waited) break;
            if (mm < p.M) {
                uint16_t* yrow = p.Y + (int64_t)mm * p.N + n_tile * 256 + 128 * half;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn(v[8 * c + 2 * u], sc));
                        const __nv_bfloat16 hi = __float2bfloat16_rn(__fmul_rn(v[8 * c + 2 * u + 1], sc));
                        w[u] = (uint32_t)(*reinterpret_cast<const uint16_t*>(&lo)) |
                               ((uint32_t)(*reinterpret_cast<const uint16_t*>(&hi)) << 16);
                    }
                    *reinterpret_cast<uint4*>(yrow + 8 * c) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    }
    // the pair's MMAs read both CTAs' shared memory and write both tensor memories: neither
    // CTA releases its tensor memory or exits before both are done
    tc_fence_before();
    __syncwarp();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::kTmemCols);
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
    if (s > kMaxSplits) s = kMaxSplits;
    if (s > KS) s = KS;
    d.iters = (KS + s - 1) / s;
    d.splits = (KS + d.iters - 1) / d.iters;
    d.cluster = d.splits > 1 && d.splits <= kMaxClusterSplits;
    return d;
}

size_t decode_workspace_bytes(int M, int N, int K) {
    DecodePlan d = plan_decode(M, N, K);
    if (d.splits <= 1 || d.cluster) return 0;
    size_t part = (size_t)d.splits * d.tiles_m * d.BN * N * sizeof(float);
    part = (part + 255) & ~size_t(255);
    return part + (size_t)d.tiles_m * d.tiles_n * sizeof(int);
}

template <int BN>
static cudaError_t launch_decode_bn(const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                                   const DecodePlan& d, cudaStream_t s) {
    using C = DecodeCfg<BN>;
    static std::atomic<bool> attr_set[64];
    cudaError_t e = once_per_device(attr_set, [] {
        return cudaFuncSetAttribute(k_gemm_decode<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    dim3 grid(d.tiles_n, d.splits, d.tiles_m);
    return launch_pdl(k_gemm_decode<BN>, grid, dim3(C::kThreads), C::kSmemBytes, s, d.cluster ? d.splits : 1, tw, tx,
                      p);
}

cudaError_t launch_gemm_decode(const CUtensorMap& tw, const CUtensorMap& tx, GemmParams p, const DecodePlan& d,
                               cudaStream_t s) {
    p.splits = d.splits;
    p.iters_per_split = d.iters;
    p.cluster = d.cluster ? 1 : 0;
    switch (d.BN) {
        case 16: return launch_decode_bn<16>(tw, tx, p, d, s);
        case 32: return launch_decode_bn<32>(tw, tx, p, d, s);
        case 64: return launch_decode_bn<64>(tw, tx, p, d, s);
        default: return launch_decode_bn<128>(tw, tx, p, d, s);
    }
}

static int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || sms <= 0) {
        cudaGetLastError();
        return 148;
    }
    return sms;
}

StreamKPlan plan_streamk(int M, int N, int K) {
    StreamKPlan d;
    d.BN = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
    d.tiles_m = (M + d.BN - 1) / d.BN;
    d.tiles_n = N / 128;
    const int KS = K / 256;
    const int64_t tiles = (int64_t)d.tiles_m * d.tiles_n;
    const int64_t units = tiles * KS;
    d.units = (int)units;
    d.grid = (int)std::min<int64_t>(units, device_sms());
    // a tile is split when its first and last units belong to different CTAs
    bool split = false;
    auto owner = [&](int64_t u) { return ((u + 1) * d.grid - 1) / units; };
    for (int64_t t = 0; t < tiles && !split; ++t) split = owner(t * KS) != owner((t + 1) * KS - 1);
    d.slots_bytes = split ? (((size_t)2 * d.grid * d.BN * 128 * sizeof(float) + 255) & ~size_t(255)) : 0;
    d.ws = split ? d.slots_bytes + (size_t)tiles * sizeof(int) : 0;
    return d;
}

template <int BN>
static cudaError_t launch_streamk_bn(const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                                     const StreamKPlan& d, cudaStream_t s) {
    using C = SKCfg<BN>;
    static std::atomic<bool> attr_set[64];
    cudaError_t e = once_per_device(attr_set, [] {
        return cudaFuncSetAttribute(k_gemm_streamk<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    return launch_pdl(k_gemm_streamk<BN>, dim3(d.grid), dim3(C::kThreads), C::kSmemBytes, s, 1, tw, tx, p);
}

cudaError_t launch_gemm_streamk(const CUtensorMap& tw, const CUtensorMap& tx, GemmParams p, const StreamKPlan& d,
                                cudaStream_t s) {
    p.units = d.units;
    p.tiles_m = d.tiles_m;
    p.tiles_n = d.tiles_n;
    switch (d.BN) {
        case 16: return launch_streamk_bn<16>(tw, tx, p, d, s);
        case 32: return launch_streamk_bn<32>(tw, tx, p, d, s);
        case 64: return launch_streamk_bn<64>(tw, tx, p, d, s);
        default: return launch_streamk_bn<128>(tw, tx, p, d, s);
    }
}

}  // namespace mq

extern "C" mq_status mq_timeline_read(void* out, size_t bytes) {
#ifdef MQ_TIMELINE
    if (!out || bytes < sizeof(mq::g_timeline)) return MQ_ERR_INVALID_ARG;
    if (cudaMemcpyFromSymbol(out, mq::g_timeline, sizeof(mq::g_timeline)) != cudaSuccess) return MQ_ERR_CUDA;
    static const unsigned long long zero[MQ_TIMELINE_CTAS][MQ_TIMELINE_EVENTS] = {};
    return cudaMemcpyToSymbol(mq::g_timeline, zero, sizeof(zero)) == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
#else
    (void)out;
    (void)bytes;
    return MQ_ERR_INVALID_ARG;
#endif
}

namespace mq {
// Device address of the error word (for kernels of other translation units).
cudaError_t error_word(int** ptr) { return cudaGetSymbolAddress(reinterpret_cast<void**>(ptr), g_error); }

int plan_small(int M, int N, int K) {
    if (M > 32) return 0;
    const int tiles = N / 128, KS = K / 256, sms = device_sms();
    if (2 * tiles > sms) return 0;  // enough tiles to keep every SM streaming: stream-K
    int S = sms / tiles;
    if (S > 8) S = 8;
    if (S > KS) S = KS;
    if ((KS + S - 1) / S > 8) return 0;  // long K ranges stream better through the deep ring
    return S;
}

template <int BN>
static cudaError_t launch_small_bn(const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p, int S,
                                   cudaStream_t s) {
    using C = SmallCfg<BN>;
    static std::atomic<bool> attr_set[64];
    cudaError_t e = once_per_device(attr_set, [] {
        return cudaFuncSetAttribute(k_gemm_small<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    const int tiles = p.N / 128;
    return launch_pdl_cluster(k_gemm_small<BN>, dim3(tiles * S), dim3(C::kThreads), C::kSmemBytes, s, dim3(S, 1, 1),
                              tw, tx, p);
}

cudaError_t launch_gemm_small(const CUtensorMap& tw, const CUtensorMap& tx, GemmParams p, int S, cudaStream_t s) {
    p.splits = S;
    p.tiles_m = 1;
    p.tiles_n = p.N / 128;
    return p.M <= 16 ? launch_small_bn<16>(tw, tx, p, S, s) : launch_small_bn<32>(tw, tx, p, S, s);
}

cudaError_t launch_gemm_prefill2(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& twsf,
                                 const CUtensorMap& txsf, const CUtensorMap& trc, const CUtensorMap& trsf,
                                 const GemmParams& p, cudaStream_t s) {
    static std::atomic<bool> attr_set[64];
    cudaError_t e = once_per_device(attr_set, [] {
        return cudaFuncSetAttribute(k_gemm_prefill2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Prefill2Cfg::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    const int pairs_max = device_sms() / 2;
    const int ntiles = ((p.M + 255) / 256) * (p.N / 256);
    const int pairs = ntiles < pairs_max ? ntiles : pairs_max;
    return launch_pdl_cluster(k_gemm_prefill2, dim3(2 * pairs), dim3(Prefill2Cfg::kThreads), Prefill2Cfg::kSmemBytes,
                              s, dim3(2, 1, 1), tw, tx, twsf, txsf, trc, trsf, p);
}

cudaError_t read_clear_error(int* value) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_error, sizeof(int));
    if (e != cudaSuccess || *value == 0) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_error, &zero, sizeof(int));
}

}  // namespace mq

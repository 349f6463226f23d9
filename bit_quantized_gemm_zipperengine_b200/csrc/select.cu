// Block-wise residual allocation (MosaicQuant summary, "Methodology" section 2):
// the Hessian-guided Delta-score of every 64x64 weight block, top-K selection at a
// block budget, and packing of the selected residual blocks for the fused GEMM.
#include "common.cuh"
#include "nvfp4.cuh"
#include "quant.cuh"

namespace mq {

// ------------------------------------------------------------------ Delta-score
// Persistent CTAs (8 warps) walk over strips of two vertically adjacent 64x64 blocks
// (block rows 2i and 2i+1, block column kt); TMA stages each strip's bf16 tile (128 rows
// x 128 bytes, 128-byte swizzle; rows past N read as zero) into a ring of shared-memory
// buffers ahead of the arithmetic. Warp w works on block w / 4 of the strip and its group
// column q = w % 4 (16 K elements); lane r owns the block's rows r and r+32, so the first
// level of the fixed pairwise row tree (v[i] += v[i+32]) happens in registers. The
// remaining levels (+16, +8, +4, +2, +1) run as a butterfly over the lanes that at each
// level also halves the set of columns a lane keeps: the adds are exactly the tree's
// pairs, and at the end lanes 2c and 2c+1 hold column c of the group. e and e' are
// recomputed from W and the tensor scale with the weight quantizer's arithmetic, so they
// are bit-identical to the stored codes.
// tau = fp64(e)^2 - fp64(e')^2 (both squares exact in fp64, one rounding), the row tree,
// p_k = H_k c_k and the 64-column tree all in fp64.
// Codes and scales are gathered in shared memory and written as whole 32-byte sectors:
// a strip's 128 rows x 32 bytes of codes, and its 512-byte chunk of the GEMM's tiled scale
// layout (one 128-row tile x 4 groups) at once.
constexpr int kQDStages = 3;
constexpr int kQDRows = 128;                   // rows of a strip
constexpr int kQDTile = kQDRows * 128;         // bytes of one staged strip
constexpr int kQDThreads = 256;
constexpr int kQDStageOff = kQDStages * kQDTile;
// staging after the tiles: codes [128][32], residual codes [128][32], tiled scales [512],
// linear scales [128][4] and residual linear scales [128][4], column products [2][64]
constexpr int kQDOffC = kQDStageOff, kQDOffRC = kQDOffC + 4096, kQDOffSw = kQDOffRC + 4096;
constexpr int kQDOffSl = kQDOffSw + 512, kQDOffRSl = kQDOffSl + 512, kQDOffP = kQDOffRSl + 512;
constexpr int kQDOffBar = kQDOffP + 2 * 64 * 8;
constexpr size_t kQDSmem = kQDOffBar + 64 + 1024;

// 16 values of row rl, group q of a staged tile (16-byte chunk c of a row sits at
// chunk position c ^ (rl % 8): the TMA 128-byte swizzle).
__device__ __forceinline__ void tile_group(const uint8_t* tile, int rl, int q, float (&a)[16]) {
    const uint4* row = reinterpret_cast<const uint4*>(tile + rl * 128);
    const uint4 v0 = row[(2 * q) ^ (rl & 7)], v1 = row[(2 * q + 1) ^ (rl & 7)];
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        a[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        a[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
}

// One strip: quantization (when kWriteCodes), Delta of its one or two blocks, and the
// coalesced stores. `nblk_rows` = N / 64.
template <bool kWriteCodes, bool kWriteResid>
__device__ __forceinline__ void quant_delta_strip(const uint8_t* tile, uint8_t* st, int K, int nblk_rows,
                                                  const float* __restrict__ H, float g, const float2* tab, int si,
                                                  int kt,
                                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                  uint8_t* __restrict__ sf_swz, uint8_t* __restrict__ rcodes,
                                                  uint8_t* __restrict__ rsf, double* __restrict__ delta) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = warp >> 2, q = warp & 3;
    const int KB = K / 64;
    const float g6 = __fmul_rn(6.0f, g);
    double* pcol = reinterpret_cast<double*>(st + kQDOffP) + blk * 64;
    double v[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rl = blk * 64 + lane + 32 * h;  // strip row
        float a[16];
        tile_group(tile, rl, q, a);
        float deq[16], R[16], rdeq[16];
        uint32_t lo, hi, rlo, rhi;
        const uint32_t sfb = nvfp4_group_tab(a, g6, tab, lo, hi, deq);
#pragma unroll
        for (int i = 0; i < 16; ++i) R[i] = __fsub_rn(a[i], deq[i]);
        const uint32_t rsb = nvfp4_group_tab(R, g6, tab, rlo, rhi, rdeq);
        if (kWriteCodes) {
            *reinterpret_cast<uint2*>(st + kQDOffC + rl * 32 + q * 8) = make_uint2(lo, hi);
            st[kQDOffSw + (rl & 31) * 16 + (rl >> 5) * 4 + q] = (uint8_t)sfb;
            st[kQDOffSl + rl * 4 + q] = (uint8_t)sfb;
        }
        if (kWriteResid) {
            *reinterpret_cast<uint2*>(st + kQDOffRC + rl * 32 + q * 8) = make_uint2(rlo, rhi);
            st[kQDOffRSl + rl * 4 + q] = (uint8_t)rsb;
        }
        // tau = fp64(e)^2 - fp64(e')^2 with e = R, e' = R - deqR: e'^2 is exact in fp64, so
        // the fused multiply-add rounds only the difference, as e*e - e'*e' does
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const double e = (double)R[j], f = (double)__fsub_rn(R[j], rdeq[j]);
            const double t = __fma_rn(e, e, -__dmul_rn(f, f));
            v[j] = h ? __dadd_rn(v[j], t) : t;
        }
    }
    // butterfly: masks 16, 8, 4, 2 keep n = 8, 4, 2, 1 columns; then mask 1 adds pairs
#pragma unroll
    for (int m = 16, n = 8; m >= 2; m >>= 1, n >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int j = 0; j < n; ++j) {
            const double send = upper ? v[j] : v[j + n];
            const double keep = upper ? v[j + n] : v[j];
            v[j] = __dadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, m));
        }
    }
    const double colsum = __dadd_rn(v[0], __shfl_xor_sync(0xffffffffu, v[0], 1));
    const int c = (lane >> 1) & 15;
    if ((lane & 1) == 0) pcol[q * 16 + c] = __dmul_rn((double)__ldg(H + kt * 64 + q * 16 + c), colsum);
    __syncthreads();
    const int nt = 2 * si + blk;
    if (q == 0 && nt < nblk_rows) {  // warps 0 and 4: the 64-column tree of their block
        double d = __dadd_rn(pcol[lane], pcol[lane + 32]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d = __dadd_rn(d, __shfl_down_sync(0xffffffffu, d, o));
        if (lane == 0) delta[(int64_t)nt * KB + kt] = d;
    }
    const int rows = min(kQDRows, (nblk_rows - 2 * si) * 64);  // rows of the strip inside W
    const int t = threadIdx.x;
    if (kWriteCodes) {
        {   // codes: thread t writes half t % 2 of row t / 2 (two lanes make one sector)
            const int r = t >> 1;
            if (r < rows)
                *reinterpret_cast<uint4*>(codes + (int64_t)(si * kQDRows + r) * (K / 2) + kt * 32 + 16 * (t & 1)) =
                    *reinterpret_cast<const uint4*>(st + kQDOffC + r * 32 + 16 * (t & 1));
        }
        if (t < 32)  // the strip's 512-byte chunk of the tiled layout (rows past N: scale 0)
            *reinterpret_cast<uint4*>(sf_swz + ((int64_t)si * KB + kt) * 512 + 16 * t) =
                *reinterpret_cast<const uint4*>(st + kQDOffSw + 16 * t);
        if (sf && t < rows)
            *reinterpret_cast<uint32_t*>(sf + (int64_t)(si * kQDRows + t) * (K / 16) + kt * 4) =
                *reinterpret_cast<const uint32_t*>(st + kQDOffSl + 4 * t);
    }
    if (kWriteResid) {
        const int r = t >> 1;
        if (r < rows)
            *reinterpret_cast<uint4*>(rcodes + (int64_t)(si * kQDRows + r) * (K / 2) + kt * 32 + 16 * (t & 1)) =
                *reinterpret_cast<const uint4*>(st + kQDOffRC + r * 32 + 16 * (t & 1));
        if (t < rows)
            *reinterpret_cast<uint32_t*>(rsf + (int64_t)(si * kQDRows + t) * (K / 16) + kt * 4) =
                *reinterpret_cast<const uint32_t*>(st + kQDOffRSl + 4 * t);
    }
}

// Activation rows the whole-path call hands to the quantize+Delta kernel (act.rows == 0:
// none). The CTAs with the fewest strips take them after their strips, one row per CTA
// at a time, so the rows fill the pass's tail instead of following it. K <= 16 x threads.
struct ActRows {
    const uint16_t* X;
    int M, rows;  // rows: M padded to a multiple of 128 (rows >= M clear their scales)
    uint8_t* codes;
    uint8_t* sf;
    uint8_t* sf_swz;
    float* g_x;
};

// kWriteCodes = false: Delta only, tensor scale read from g_in. kWriteCodes = true: base
// codes and scales, Delta, and (kWriteResid) the full residual, in one pass over W; the
// tensor scale comes from the |W| maximum partials. Persistent: CTA c handles strips c,
// c + gridDim.x, ... in (strip row, kt) order, kt fastest; then activation rows (act).
template <bool kWriteCodes, bool kWriteResid>
__global__ void __launch_bounds__(kQDThreads, 3) k_quant_delta(const __grid_constant__ CUtensorMap tmap_w, int N, int K,
                                                            const float* __restrict__ H, const float* __restrict__ g_in,
                                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                            uint8_t* __restrict__ sf_swz, float* __restrict__ g_out,
                                                            uint8_t* __restrict__ rcodes, uint8_t* __restrict__ rsf,
                                                            double* __restrict__ delta, int* __restrict__ err,
                                                            const ActRows act) {
    extern __shared__ uint8_t qd_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qd_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kQDOffBar);
    const int KB = K / 64, nbr = N / 64, nstrips = ((nbr + 1) / 2) * KB;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQDStages; ++s) mbar_init(&full[s], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmap_w);
    }
    __syncthreads();
    // this pass is the last full read of W (the weight maxima pass kept it in L2 for it)
    const uint64_t done = l2_policy_evict_first();
    auto issue = [&](int i) {  // strip number i of this CTA into stage i % kQDStages
        const int b = blockIdx.x + i * gridDim.x;
        if (b < nstrips) {
            const int s = i % kQDStages;
            mbar_arrive_expect_tx(&full[s], kQDTile);
            tma_load_2d_u16_hint(sm + s * kQDTile, &tmap_w, &full[s], (b % KB) * 64, (b / KB) * kQDRows, done);
        }
    };
    // W is an input of the call (never written by the preceding kernels): start loading
    if (threadIdx.x == 0)
        for (int i = 0; i < kQDStages; ++i) issue(i);
    griddep_wait();
    const float g = kWriteCodes ? tensor_scale(g_in) : __ldg(g_in);
    if (kWriteCodes && blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
    __shared__ float2 s_tab[128];  // (d, 1/d) of every scale code for this tensor scale
    nvfp4_scale_table(g, s_tab);
    __syncthreads();
    // the next kernel may start once every CTA has read the tensor-scale partials
    griddep_launch();
    bool ok = true;
    for (int i = 0;; ++i) {
        const int b = blockIdx.x + i * gridDim.x;
        if (b >= nstrips) break;
        const int s = i % kQDStages;
        if (ok) ok = mbar_wait_err(&full[s], (i / kQDStages) & 1, err);
        if (ok)
            quant_delta_strip<kWriteCodes, kWriteResid>(sm + s * kQDTile, sm, K, nbr, H, g, s_tab, b / KB, b % KB, codes,
                                                        sf, sf_swz, rcodes, rsf, delta);
        __syncthreads();  // stage s and the strip's staging are free again
        // every copy issued here is waited for by a later iteration of this loop
        if (threadIdx.x == 0 && ok) issue(i + kQDStages);
    }
    // the activation rows, the last CTAs (fewest strips) first; X is an input of the call
    for (int m = gridDim.x - 1 - blockIdx.x; m < act.rows; m += gridDim.x) {
        quant_act_row<1>(act.X, act.M, K, act.codes, act.sf, act.sf_swz, act.g_x, m);
        __syncthreads();  // the row's shared scratch is free again
    }
}

// ------------------------------------------------------------------ top-K
// Order-preserving 64-bit key of a finite double (larger value -> larger key);
// -0 is folded onto +0 so that the two tie like equal doubles do.
__device__ __forceinline__ uint64_t order_key(double d) {
    uint64_t u = (uint64_t)__double_as_longlong(d);
    if (u == 0x8000000000000000ull) u = 0;
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Exclusive block-wide sum over `kThreads` threads (returns this thread's prefix and
// the total through `total`).
template <int kThreads>
__device__ __forceinline__ int block_exclusive_sum(int v, int* scratch, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = lane < kThreads / 32 ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kThreads / 32) scratch[lane] = s;
    }
    __syncthreads();
    const int before = (warp ? scratch[warp - 1] : 0) + x - v;
    total = scratch[kThreads / 32 - 1];
    __syncthreads();
    return before;
}

constexpr int kSelThreads = 1024;
constexpr size_t kSelSmemKeysMax = 160 * 1024;
constexpr int kSelBitWords = (int)(kSelSmemKeysMax / 8 / 32);  // bitmap words of the keys that fit

constexpr int kDigitBits = 11;

// Exclusive prefix sum over the CTA's threads in thread order (kThreads <= 1024), with
// one barrier: a shuffle scan inside each warp, the warp totals through `wsum`, and the
// sum of the lower warps' totals by a warp reduction. `wsum` must not be reused before
// the next barrier.
template <int kThreads>
__device__ __forceinline__ int block_excl_sum_1bar(int v, int* wsum) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    const int ws = (lane < kThreads / 32 && lane < warp) ? wsum[lane] : 0;
    return (int)__reduce_add_sync(0xffffffffu, (unsigned)ws) + x - v;
}

// Top-K selection, one CTA of 1024 threads:
//  1. keys and their common leading bits (eight loads in flight per thread when the keys
//     do not fit in shared memory and are read again from global memory in every pass);
//  2. radix passes of up to 11 bits below the common prefix narrow the bucket that holds
//     the budget-th largest key until the bucket is taken whole (its count equals the
//     keys still needed) or is a single key value;
//  3. compaction in block order, warp w over the contiguous index range w: every key above
//     the bucket, and the bucket's keys (all of them, or the lowest-index `need` ones of a
//     single key value), which writes sel ascending.
// rank (the selected blocks in Delta order) comes from the split counting rank CTAs.
template <bool kSmemKeys>
__global__ void __launch_bounds__(kSelThreads) k_topk_large(const double* __restrict__ delta, int B, int budget,
                                                            int32_t* __restrict__ sel) {
    extern __shared__ __align__(16) uint64_t dyn[];
    uint64_t* keys = dyn;  // [B] when kSmemKeys
    __shared__ unsigned hist[2][1 << kDigitBits];  // pass p counts into hist[p % 2]
    __shared__ uint32_t s_gtw[kSelBitWords], s_eqw[kSelBitWords];
    __shared__ uint32_t s_and[64], s_or[64];
    __shared__ uint64_t s_prefix;
    __shared__ int s_pos, s_need, s_cand;
    __shared__ int s_gt[32], s_eq[32], s_base[32], s_eqb[32];
    __shared__ int scratch[32], scratch2[32];
    griddep_wait();  // Delta comes from the previous kernel
    griddep_launch();
    constexpr int U = 8;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto key_of = [&](int i) -> uint64_t { return kSmemKeys ? keys[i] : order_key(delta[i]); };

    uint64_t a = ~0ull, o = 0ull;
    for (int i0 = tid; i0 < B; i0 += U * kSelThreads) {
        double d[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * kSelThreads;
            d[u] = i < B ? delta[i] : 0.0;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * kSelThreads;
            if (i < B) {
                const uint64_t k = order_key(d[u]);
                if (kSmemKeys) keys[i] = k;
                a &= k;
                o |= k;
            }
        }
    }
    {
        const uint32_t ah = __reduce_and_sync(0xffffffffu, (uint32_t)(a >> 32));
        const uint32_t al = __reduce_and_sync(0xffffffffu, (uint32_t)a);
        const uint32_t oh = __reduce_or_sync(0xffffffffu, (uint32_t)(o >> 32));
        const uint32_t ol = __reduce_or_sync(0xffffffffu, (uint32_t)o);
        if (lane == 0) {
            s_and[2 * warp] = ah;
            s_and[2 * warp + 1] = al;
            s_or[2 * warp] = oh;
            s_or[2 * warp + 1] = ol;
        }
    }
    for (int b = tid; b < (1 << kDigitBits); b += kSelThreads) hist[0][b] = 0;
    __syncthreads();
    if (warp == 0) {
        const uint32_t ah = __reduce_and_sync(0xffffffffu, s_and[2 * lane]);
        const uint32_t al = __reduce_and_sync(0xffffffffu, s_and[2 * lane + 1]);
        const uint32_t oh = __reduce_or_sync(0xffffffffu, s_or[2 * lane]);
        const uint32_t ol = __reduce_or_sync(0xffffffffu, s_or[2 * lane + 1]);
        a = ((uint64_t)ah << 32) | al;
        o = ((uint64_t)oh << 32) | ol;
        if (lane == 0) {
            const int cp = (a ^ o) ? __clzll((long long)(a ^ o)) : 64;
            s_pos = 64 - cp;
            s_prefix = cp ? (a & (~0ull << (64 - cp))) : 0ull;
            s_need = budget;
            s_cand = B;
        }
    }
    __syncthreads();
    for (int pass = 0; s_pos > 0 && s_cand > s_need; ++pass) {
        const int pos = s_pos, w = pos < kDigitBits ? pos : kDigitBits, shift = pos - w;
        const uint64_t prefix = s_prefix, hi = pos >= 64 ? 0ull : (~0ull << pos);
        const int need = s_need;
        const int nb = 1 << w;
        unsigned* h = hist[pass & 1];
        // the other buffer (read by the previous pass's scan, which every thread has left)
        // is cleared for the next pass
        for (int b = tid; b < (1 << kDigitBits); b += kSelThreads) hist[(pass + 1) & 1][b] = 0;
        for (int i0 = tid - lane; i0 < B; i0 += U * kSelThreads) {  // warp-uniform
            uint64_t k[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + lane + u * kSelThreads;
                k[u] = i < B ? key_of(i) : 0ull;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + lane + u * kSelThreads;
                unsigned digit = 1u << kDigitBits;  // not counted
                if (i < B && (k[u] & hi) == prefix) digit = (unsigned)(k[u] >> shift) & (nb - 1);
                if (digit < (1u << kDigitBits)) atomicAdd(&h[digit], 1u);
            }
        }
        __syncthreads();
        const int b0 = nb - 1 - 2 * tid;
        const unsigned c0 = b0 >= 0 ? h[b0] : 0u, c1 = b0 - 1 >= 0 ? h[b0 - 1] : 0u;
        const int above = block_excl_sum_1bar<kSelThreads>((int)(c0 + c1), scratch);
        if (b0 >= 0 && above < need && above + (int)(c0 + c1) >= need) {
            const bool first = above + (int)c0 >= need;
            const int digit = first ? b0 : b0 - 1;
            s_need = need - (first ? above : above + (int)c0);
            s_cand = (int)(first ? c0 : c1);
            s_prefix = prefix | ((uint64_t)digit << shift);
            s_pos = shift;
        }
        __syncthreads();
    }
    const int pos = s_pos, need = s_need;
    const bool whole = s_cand == s_need;
    const uint64_t prefix = s_prefix, hi = pos >= 64 ? 0ull : (~0ull << pos);
    if (kSmemKeys) {
        // the keys above the bucket and in it as bitmaps (warp ballots over 32-key words),
        // then thread t turns word t into sel entries at the count of selected keys before it
        const int nw = (B + 31) >> 5;
        for (int wd = warp; wd < nw; wd += 32) {
            const int i = wd * 32 + lane;
            const bool valid = i < B;
            const uint64_t t = valid ? (keys[i] & hi) : 0ull;
            const unsigned g = __ballot_sync(0xffffffffu, valid && t > prefix);
            const unsigned e = __ballot_sync(0xffffffffu, valid && t == prefix);
            if (lane == 0) {
                s_gtw[wd] = g;
                s_eqw[wd] = e;
            }
        }
        __syncthreads();
        const uint32_t g = tid < nw ? s_gtw[tid] : 0u, e = tid < nw ? s_eqw[tid] : 0u;
        uint32_t take = g;
        if (whole) {
            take |= e;
        } else {  // one tied value: its lowest-index `need` keys
            int left = need - block_excl_sum_1bar<kSelThreads>(__popc(e), scratch2);
            for (uint32_t ee = e; left > 0 && ee; --left) {
                const uint32_t low = ee & (0u - ee);
                take |= low;
                ee ^= low;
            }
        }
        int out = block_excl_sum_1bar<kSelThreads>(__popc(take), scratch);
        for (uint32_t m = take; m; m &= m - 1) sel[out++] = tid * 32 + (__ffs(m) - 1);
        return;
    }
    const int CW = (B + 32 * 32 - 1) / (32 * 32) * 32;  // indices per warp, a multiple of 32
    const int w0 = min(B, warp * CW), w1 = min(B, w0 + CW);
    int gt = 0, eq = 0;
    for (int i0 = w0; i0 < w1; i0 += 32 * U) {
        uint64_t k[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + lane + 32 * u;
            k[u] = i < w1 ? key_of(i) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + lane + 32 * u;
            if (i < w1) {
                const uint64_t t = k[u] & hi;
                gt += t > prefix;
                eq += t == prefix;
            }
        }
    }
    gt = (int)__reduce_add_sync(0xffffffffu, (unsigned)gt);
    eq = (int)__reduce_add_sync(0xffffffffu, (unsigned)eq);
    if (lane == 0) {
        s_gt[warp] = gt;
        s_eq[warp] = eq;
    }
    __syncthreads();
    if (warp == 0) {
        const int g = s_gt[lane], e = s_eq[lane];
        int ie = e;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, ie, d);
            if (lane >= d) ie += y;
        }
        const int eqb = ie - e;
        const int take = whole ? e : max(0, min(e, need - eqb));
        int it = g + take;
        const int t0 = it;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, it, d);
            if (lane >= d) it += y;
        }
        s_eqb[lane] = eqb;
        s_base[lane] = it - t0;
    }
    __syncthreads();
    int out = s_base[warp], eq_seen = s_eqb[warp];
    const unsigned lt = (1u << lane) - 1u;
    for (int i0 = w0; i0 < w1; i0 += 32 * U) {
        uint64_t k[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + lane + 32 * u;
            k[u] = i < w1 ? key_of(i) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + lane + 32 * u;
            const bool valid = i < w1;
            const uint64_t t = k[u] & hi;
            const bool is_gt = valid && t > prefix, is_eq = valid && t == prefix;
            const unsigned meq = __ballot_sync(0xffffffffu, is_eq);
            bool take = is_gt;
            if (is_eq) take = whole || eq_seen + __popc(meq & lt) < need;
            eq_seen += __popc(meq);
            const unsigned mt = __ballot_sync(0xffffffffu, take);
            if (take) sel[out + __popc(mt & lt)] = i;
            out += __popc(mt);
        }
    }
}

// Top-K selection for more keys than one CTA's shared memory holds: a cluster of C CTAs
// (one cluster, grid == cluster), CTA c holding the keys of blocks [c chunk, (c+1) chunk)
// in its shared memory (chunk a multiple of 32). The steps are those of k_topk_large with
// its shared-memory keys, and every decision is taken identically in every CTA from the
// same cluster-wide counts:
//  - the common leading bits from each CTA's AND / OR of its keys, read through DSMEM;
//  - in each radix pass, every CTA counts its keys into its own histogram and adds its
//    non-zero bins into the sum histogram of the bin pair's owner, CTA (b / 2) % C (remote
//    atomic adds, which do not wait for a reply); after a cluster barrier each thread reads
//    its two bins of the sum from their owner (one load) before the block scan. The sums
//    rotate over three buffers: the one a pass clears was last read two passes earlier, and
//    every CTA has crossed the previous pass's cluster barrier since;
//  - compaction: each CTA's counts above the bucket and in it are exchanged once, giving its
//    offset in sel and the tied keys that the lower CTAs take; a last cluster barrier keeps
//    every CTA resident until the others have read its counts.
constexpr int kTkMaxCluster = 8;
constexpr int kTkCtaKeys = 20480;  // keys one CTA holds (160 KB)

__global__ void __launch_bounds__(kSelThreads) k_topk_cluster(const double* __restrict__ delta, int B, int budget,
                                                              int chunk, int32_t* __restrict__ sel) {
    extern __shared__ __align__(16) uint64_t dyn[];
    uint64_t* keys = dyn;  // [chunk]
    __shared__ unsigned hist[1 << kDigitBits];        // this CTA's counts of the pass
    __shared__ __align__(8) unsigned hsum[3][1 << kDigitBits];  // the cluster's counts of owned bins
    __shared__ uint32_t s_gtw[kTkCtaKeys / 32], s_eqw[kTkCtaKeys / 32];
    __shared__ uint32_t s_and[64], s_or[64];
    __shared__ uint64_t s_ao[2];   // this CTA's AND and OR of its keys (read by the cluster)
    __shared__ int s_cnt[2];       // this CTA's keys above the bucket and in it (read by the cluster)
    __shared__ int s_out0, s_eqb;  // this CTA's first sel entry; tied keys taken by lower CTAs
    __shared__ uint64_t s_prefix;
    __shared__ int s_pos, s_need, s_cand;
    __shared__ int scratch[32], scratch2[32];
    griddep_wait();  // Delta comes from the previous kernel
    griddep_launch();
    constexpr int U = 8;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = (int)gridDim.x, c = (int)cluster_ctarank();
    const int base = c * chunk, n = max(0, min(chunk, B - base));

    uint64_t a = ~0ull, o = 0ull;
    for (int i0 = tid; i0 < n; i0 += U * kSelThreads) {
        double d[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * kSelThreads;
            d[u] = i < n ? delta[base + i] : 0.0;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * kSelThreads;
            if (i < n) {
                const uint64_t k = order_key(d[u]);
                keys[i] = k;
                a &= k;
                o |= k;
            }
        }
    }
    {
        const uint32_t ah = __reduce_and_sync(0xffffffffu, (uint32_t)(a >> 32));
        const uint32_t al = __reduce_and_sync(0xffffffffu, (uint32_t)a);
        const uint32_t oh = __reduce_or_sync(0xffffffffu, (uint32_t)(o >> 32));
        const uint32_t ol = __reduce_or_sync(0xffffffffu, (uint32_t)o);
        if (lane == 0) {
            s_and[2 * warp] = ah;
            s_and[2 * warp + 1] = al;
            s_or[2 * warp] = oh;
            s_or[2 * warp + 1] = ol;
        }
    }
    for (int b = tid; b < (1 << kDigitBits); b += kSelThreads) hsum[0][b] = 0;
    __syncthreads();
    if (warp == 0) {
        const uint32_t ah = __reduce_and_sync(0xffffffffu, s_and[2 * lane]);
        const uint32_t al = __reduce_and_sync(0xffffffffu, s_and[2 * lane + 1]);
        const uint32_t oh = __reduce_or_sync(0xffffffffu, s_or[2 * lane]);
        const uint32_t ol = __reduce_or_sync(0xffffffffu, s_or[2 * lane + 1]);
        if (lane == 0) {
            s_ao[0] = ((uint64_t)ah << 32) | al;
            s_ao[1] = ((uint64_t)oh << 32) | ol;
        }
    }
    cluster_sync();  // every CTA's AND / OR, and the first sum histogram cleared
    if (warp == 0) {
        const uint64_t ar = lane < C ? ld_dsmem_u64(&s_ao[0], lane) : ~0ull;
        const uint64_t orr = lane < C ? ld_dsmem_u64(&s_ao[1], lane) : 0ull;
        const uint32_t ah = __reduce_and_sync(0xffffffffu, (uint32_t)(ar >> 32));
        const uint32_t al = __reduce_and_sync(0xffffffffu, (uint32_t)ar);
        const uint32_t oh = __reduce_or_sync(0xffffffffu, (uint32_t)(orr >> 32));
        const uint32_t ol = __reduce_or_sync(0xffffffffu, (uint32_t)orr);
        a = ((uint64_t)ah << 32) | al;
        o = ((uint64_t)oh << 32) | ol;
        if (lane == 0) {
            const int cp = (a ^ o) ? __clzll((long long)(a ^ o)) : 64;
            s_pos = 64 - cp;
            s_prefix = cp ? (a & (~0ull << (64 - cp))) : 0ull;
            s_need = budget;
            s_cand = B;
        }
    }
    __syncthreads();
    for (int pass = 0; s_pos > 0 && s_cand > s_need; ++pass) {  // identical in every CTA
        const int pos = s_pos, w = pos < kDigitBits ? pos : kDigitBits, shift = pos - w;
        const uint64_t prefix = s_prefix, hi = pos >= 64 ? 0ull : (~0ull << pos);
        const int need = s_need;
        const int nb = 1 << w;
        unsigned* h = hist;
        unsigned* hs = hsum[pass % 3];
        for (int b = tid; b < (1 << kDigitBits); b += kSelThreads) {
            h[b] = 0;
            hsum[(pass + 1) % 3][b] = 0;
        }
        __syncthreads();
        for (int i0 = tid - lane; i0 < n; i0 += U * kSelThreads) {  // warp-uniform
            uint64_t k[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + lane + u * kSelThreads;
                k[u] = i < n ? keys[i] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + lane + u * kSelThreads;
                if (i < n && (k[u] & hi) == prefix) atomicAdd(&h[(unsigned)(k[u] >> shift) & (nb - 1)], 1u);
            }
        }
        __syncthreads();  // this CTA's counts are complete
        const int b0 = nb - 1 - 2 * tid;
        // bins b0 - 1 and b0 (b0 odd: nb is even) belong to CTA (b0 / 2) % C
        const uint32_t owner = b0 >= 0 ? (uint32_t)((b0 >> 1) % C) : 0u;
        if (b0 >= 1) {
            const unsigned v0 = h[b0], v1 = h[b0 - 1];
            if (v0) red_add_dsmem_u32(mapa_u32(smem_u32(&hs[b0]), owner), v0);
            if (v1) red_add_dsmem_u32(mapa_u32(smem_u32(&hs[b0 - 1]), owner), v1);
        }
        cluster_sync();  // the cluster's counts of this pass are complete at their owners
        unsigned c0 = 0u, c1 = 0u;
        if (b0 >= 1) {
            const uint2 v = ld_dsmem_u32x2(&hs[b0 - 1], owner);
            c0 = v.y;
            c1 = v.x;
        }
        const int above = block_excl_sum_1bar<kSelThreads>((int)(c0 + c1), scratch);
        if (b0 >= 0 && above < need && above + (int)(c0 + c1) >= need) {
            const bool first = above + (int)c0 >= need;
            const int digit = first ? b0 : b0 - 1;
            s_need = need - (first ? above : above + (int)c0);
            s_cand = (int)(first ? c0 : c1);
            s_prefix = prefix | ((uint64_t)digit << shift);
            s_pos = shift;
        }
        __syncthreads();
    }
    const int pos = s_pos, need = s_need;
    const bool whole = s_cand == s_need;
    const uint64_t prefix = s_prefix, hi = pos >= 64 ? 0ull : (~0ull << pos);
    // this CTA's keys above the bucket and in it, as bitmaps of 32-key words
    const int nw = (n + 31) >> 5;
    for (int wd = warp; wd < nw; wd += 32) {
        const int i = wd * 32 + lane;
        const bool valid = i < n;
        const uint64_t t = valid ? (keys[i] & hi) : 0ull;
        const unsigned g = __ballot_sync(0xffffffffu, valid && t > prefix);
        const unsigned e = __ballot_sync(0xffffffffu, valid && t == prefix);
        if (lane == 0) {
            s_gtw[wd] = g;
            s_eqw[wd] = e;
        }
    }
    __syncthreads();
    const uint32_t g = tid < nw ? s_gtw[tid] : 0u, e = tid < nw ? s_eqw[tid] : 0u;
    int n_gt = 0, n_eq = 0;
    block_exclusive_sum<kSelThreads>(__popc(g), scratch, n_gt);
    const int eq_local = block_exclusive_sum<kSelThreads>(__popc(e), scratch2, n_eq);
    if (tid == 0) {
        s_cnt[0] = n_gt;
        s_cnt[1] = n_eq;
    }
    cluster_sync();  // every CTA's counts
    if (warp == 0) {
        const int gr = lane < C ? (int)ld_dsmem_u32(&s_cnt[0], lane) : 0;
        const int er = lane < C ? (int)ld_dsmem_u32(&s_cnt[1], lane) : 0;
        int ie = er;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, ie, d);
            if (lane >= d) ie += y;
        }
        const int eqb = ie - er;  // tied keys in the lower CTAs
        const int take = whole ? er : max(0, min(er, need - eqb));
        int it = gr + take;
        const int t0 = it;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, it, d);
            if (lane >= d) it += y;
        }
        if (lane == c) {
            s_out0 = it - t0;
            s_eqb = eqb;
        }
    }
    cluster_sync();  // no CTA leaves while another still reads its counts
    uint32_t take = g;
    if (whole) {
        take |= e;
    } else {  // one tied value: its lowest-index `need` keys over the whole cluster
        int left = need - s_eqb - eq_local;
        for (uint32_t ee = e; left > 0 && ee; --left) {
            const uint32_t low = ee & (0u - ee);
            take |= low;
            ee ^= low;
        }
    }
    int out = s_out0 + block_excl_sum_1bar<kSelThreads>(__popc(take), scratch);
    for (uint32_t m = take; m; m &= m - 1) sel[out++] = base + tid * 32 + (__ffs(m) - 1);
}

// rank: position of selected block i = #{j : key_j > key_i} + #{j < i : key_j == key_i}
// over the selected set (sel ascending, so a lower list index is a lower block index),
// that is #{j < i : key_j >= key_i} + #{j > i : key_j > key_i}. A CTA of 4 warps owns the
// 32 selected blocks 32 c .. 32 c + 31, eight per warp, whose keys every lane keeps in
// registers; it stages the selected keys in tiles of 2048, and lane l compares every 32nd
// key of a tile with its warp's eight (one shared-memory load per eight comparisons). A
// tile wholly before (after) the CTA's blocks needs only the >= (>) test.
constexpr int kRankTile = 2048;
constexpr int kRankPerWarp = 8;
constexpr int kRankPerCta = 4 * kRankPerWarp;  // 128 threads
__device__ __forceinline__ void rank_split_cta(const double* __restrict__ delta, const int32_t* __restrict__ sel,
                                               int budget, int32_t* __restrict__ rank, int c) {
    __shared__ uint64_t tk[kRankTile];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int c0 = c * kRankPerCta, c1 = min(budget, c0 + kRankPerCta);
    const int i0 = c0 + warp * kRankPerWarp;
    uint64_t mine[kRankPerWarp];
    int cnt[kRankPerWarp];
    {
        const int i = i0 + (lane & (kRankPerWarp - 1));
        const uint64_t k = i < budget ? order_key(delta[__ldg(sel + i)]) : 0ull;
#pragma unroll
        for (int e = 0; e < kRankPerWarp; ++e) {
            mine[e] = __shfl_sync(0xffffffffu, k, e);
            cnt[e] = 0;
        }
    }
    for (int base = 0; base < budget; base += kRankTile) {
        const int n = min(kRankTile, budget - base);
        __syncthreads();  // the previous tile is no longer read
        for (int j0 = t; j0 < n; j0 += 128 * 8) {
            int sj[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + 128 * u;
                sj[u] = j < n ? __ldg(sel + base + j) : 0;
            }
            double d[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) d[u] = j0 + 128 * u < n ? delta[sj[u]] : 0.0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (j0 + 128 * u < n) tk[j0 + 128 * u] = order_key(d[u]);
        }
        __syncthreads();
        if (base + n <= c0) {  // every staged block precedes the CTA's
            for (int j = lane; j < n; j += 32) {
                const uint64_t kj = tk[j];
#pragma unroll
                for (int e = 0; e < kRankPerWarp; ++e) cnt[e] += kj >= mine[e];
            }
        } else if (base >= c1) {  // every staged block follows them
            for (int j = lane; j < n; j += 32) {
                const uint64_t kj = tk[j];
#pragma unroll
                for (int e = 0; e < kRankPerWarp; ++e) cnt[e] += kj > mine[e];
            }
        } else {
            for (int j = lane; j < n; j += 32) {
                const uint64_t kj = tk[j];
                const int g = base + j;
#pragma unroll
                for (int e = 0; e < kRankPerWarp; ++e) cnt[e] += g < i0 + e ? kj >= mine[e] : kj > mine[e];
            }
        }
    }
    int pos = 0;
#pragma unroll
    for (int e = 0; e < kRankPerWarp; ++e) {
        const int v = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt[e]);
        if (lane == e) pos = v;
    }
    if (lane < kRankPerWarp && i0 + lane < budget) rank[pos] = __ldg(sel + i0 + lane);
}

__global__ void __launch_bounds__(128) k_topk_rank_split(const double* __restrict__ delta,
                                                         const int32_t* __restrict__ sel, int budget,
                                                         int32_t* __restrict__ rank) {
    griddep_wait();
    griddep_launch();
    rank_split_cta(delta, sel, budget, rank, blockIdx.x);
}

// ------------------------------------------------------------------ pack
// Per-block-row CSR (tile_ptr) and selection bitmap of the ascending selection `sel`, one
// thread per block row nt.
__device__ __forceinline__ void pack_rows(int nt, int NBr, int KB, const int32_t* __restrict__ sel, int budget,
                                          int32_t* __restrict__ tile_ptr, uint32_t* __restrict__ bitmap) {
    const int KW = (KB + 31) / 32;
    if (nt >= NBr) return;
    auto lower_bound = [&](int key) {
        int lo = 0, hi = budget;
        while (lo < hi) {
            int mid = (lo + hi) >> 1;
            if (__ldg(sel + mid) < key) lo = mid + 1;
            else hi = mid;
        }
        return lo;
    };
    const int beg = lower_bound(nt * KB), end = lower_bound((nt + 1) * KB);
    tile_ptr[nt] = beg;
    if (nt == NBr - 1) tile_ptr[NBr] = end;
    int e = beg;
    for (int w = 0; w < KW; ++w) {
        uint32_t word = 0;
        while (e < end) {
            const int kt = __ldg(sel + e) - nt * KB;
            if ((kt >> 5) != w) break;
            word |= 1u << (kt & 31);
            ++e;
        }
        bitmap[(int64_t)nt * KW + w] = word;
    }
}

// Byte offset of packed byte j (0..31) of block row r in the MMA's no-swizzle K-major
// operand layout (8-row x 16-byte core matrices).
__device__ __forceinline__ int core_offset(int r, int j) { return (r >> 3) * 256 + (j >> 4) * 128 + (r & 7) * 16 + (j & 15); }

// CTAs [0, budget): copy selected block i into the MMA's no-swizzle K-major layout and
// its scales into the 128-row scale chunk of its band. The remaining CTAs build the
// per-block-row CSR and bitmap (one thread per block row).
__global__ void __launch_bounds__(256) k_pack(const uint8_t* __restrict__ rcodes, const uint8_t* __restrict__ rsf,
                                              int N, int K, const int32_t* __restrict__ sel, int budget,
                                              uint8_t* __restrict__ blk_codes, uint8_t* __restrict__ blk_sf,
                                              int32_t* __restrict__ blk_kt, int32_t* __restrict__ tile_ptr,
                                              uint32_t* __restrict__ bitmap) {
    griddep_wait();
    griddep_launch();
    const int KB = K / 64;
    if ((int)blockIdx.x < budget) {
        const int i = blockIdx.x;
        const int b = __ldg(sel + i), nt = b / KB, kt = b % KB;
        const int t = threadIdx.x;
        {   // codes: row r, bytes 8*c8 .. 8*c8+7 of the block row
            const int r = t >> 2, j = 8 * (t & 3);
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(rcodes + (int64_t)(nt * 64 + r) * (K / 2) + kt * 32 + j));
            *reinterpret_cast<uint2*>(blk_codes + (int64_t)i * 2048 + core_offset(r, j)) = v;
        }
        if (t < 128) {  // scales: the block's 64 rows, zeros for the other half of the band
            const int half = nt & 1;
            const int tr = t;  // tile row 0..127
            uint32_t v = 0;
            if ((tr >> 6) == half)
                v = __ldg(reinterpret_cast<const uint32_t*>(rsf + (int64_t)(nt * 64 + (tr & 63)) * (K / 16) + kt * 4));
            *reinterpret_cast<uint32_t*>(blk_sf + (int64_t)i * 512 + (tr & 31) * 16 + (tr >> 5) * 4) = v;
        }
        if (t == 0) blk_kt[i] = kt;
        return;
    }
    pack_rows((blockIdx.x - budget) * blockDim.x + threadIdx.x, N / 64, KB, sel, budget, tile_ptr, bitmap);
}

// Pack straight from W: CTAs [0, budget) recompute the residual of selected block i with
// the weight quantizer's arithmetic (base group, R = W - deq, NVFP4(R) with the same
// tensor scale), bit-identical to packing the full residual; the full residual is never
// stored. Warp q handles group column q, lane r the block rows r and r+32. The next `ncsr`
// CTAs build the CSR and bitmap; with rank != null the CTAs after them write rank (the
// selection in Delta order, which nothing downstream of the pack reads) alongside.
__global__ void __launch_bounds__(128) k_pack_w(const uint16_t* __restrict__ W, int N, int K,
                                                const float* __restrict__ g_w, const int32_t* __restrict__ sel,
                                                int budget, uint8_t* __restrict__ blk_codes,
                                                uint8_t* __restrict__ blk_sf, int32_t* __restrict__ blk_kt,
                                                int32_t* __restrict__ tile_ptr, uint32_t* __restrict__ bitmap,
                                                int ncsr, const double* __restrict__ delta,
                                                int32_t* __restrict__ rank) {
    griddep_wait();
    griddep_launch();
    const int KB = K / 64;
    if ((int)blockIdx.x >= budget + ncsr) {
        rank_split_cta(delta, sel, budget, rank, (int)blockIdx.x - budget - ncsr);
        return;
    }
    if ((int)blockIdx.x >= budget) {
        pack_rows((blockIdx.x - budget) * blockDim.x + threadIdx.x, N / 64, KB, sel, budget, tile_ptr, bitmap);
        return;
    }
    __shared__ __align__(16) uint32_t chunk[128];  // the block's positioned 512-byte scale chunk
    const int i = blockIdx.x, t = threadIdx.x, q = t >> 5, lane = t & 31;
    const int b = __ldg(sel + i), nt = b / KB, kt = b % KB;
    const float g = __ldg(g_w), g6 = __fmul_rn(6.0f, g);
    chunk[t] = 0u;
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = lane + 32 * h;
        const uint4* src = reinterpret_cast<const uint4*>(W + (int64_t)(nt * 64 + r) * K + kt * 64 + q * 16);
        const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float a[16], deq[16], R[16], rdeq[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            a[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFFu);
            a[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
        }
        uint32_t lo, hi, rlo, rhi;
        nvfp4_group(a, g, g6, lo, hi, deq);
#pragma unroll
        for (int j = 0; j < 16; ++j) R[j] = __fsub_rn(a[j], deq[j]);
        const uint32_t rsb = nvfp4_group(R, g, g6, rlo, rhi, rdeq);
        *reinterpret_cast<uint2*>(blk_codes + (int64_t)i * 2048 + core_offset(r, 8 * q)) = make_uint2(rlo, rhi);
        const int tr = 64 * (nt & 1) + r;
        reinterpret_cast<uint8_t*>(chunk)[(tr & 31) * 16 + (tr >> 5) * 4 + q] = (uint8_t)rsb;
    }
    __syncthreads();
    if (t < 32) reinterpret_cast<uint4*>(blk_sf + (int64_t)i * 512)[t] = reinterpret_cast<const uint4*>(chunk)[t];
    if (t == 0) blk_kt[i] = kt;
}

// ------------------------------------------------------------------ launchers
static int quant_delta_grid(int nstrips) {
    static std::atomic<bool> attr_set[64];
    static std::atomic<int> per_sm_cache{0};
    once_per_device(attr_set, [] {
        cudaFuncSetAttribute(k_quant_delta<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQDSmem);
        cudaFuncSetAttribute(k_quant_delta<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQDSmem);
        return cudaFuncSetAttribute(k_quant_delta<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kQDSmem);
    });
    int per_sm = per_sm_cache.load(std::memory_order_relaxed);
    if (!per_sm) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quant_delta<true, true>, kQDThreads, kQDSmem) !=
                cudaSuccess ||
            per_sm < 1)
            per_sm = 2;
        per_sm_cache.store(per_sm, std::memory_order_relaxed);
    }
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = per_sm * sms;
    return nstrips < grid ? nstrips : grid;
}

static int qd_strips(int N, int K) { return ((N / 64 + 1) / 2) * (K / 64); }

cudaError_t launch_delta(const CUtensorMap& tw, int N, int K, const float* H, const float* g, double* delta,
                         int* err, cudaStream_t s) {
    const ActRows none = {nullptr, 0, 0, nullptr, nullptr, nullptr, nullptr};
    return launch_pdl(k_quant_delta<false, false>, dim3(quant_delta_grid(qd_strips(N, K))), dim3(kQDThreads),
                      kQDSmem, s, 1, tw, N, K, H, g, (uint8_t*)nullptr, (uint8_t*)nullptr, (uint8_t*)nullptr,
                      (float*)nullptr, (uint8_t*)nullptr, (uint8_t*)nullptr, delta, err, none);
}

bool quant_delta_takes_act(int K) { return K / 16 <= kQDThreads; }

cudaError_t launch_quant_delta(const uint16_t* W, const CUtensorMap& tw, int N, int K, const float* H,
                               uint8_t* codes, uint8_t* sf, uint8_t* sf_swz, float* g, uint8_t* rcodes, uint8_t* rsf,
                               double* delta, float* partial, int* err, cudaStream_t s, const uint16_t* X, int M,
                               uint8_t* xcodes, uint8_t* xsf, uint8_t* xsf_swz, float* g_x) {
    if (X && !quant_delta_takes_act(K)) return cudaErrorInvalidValue;
    cudaError_t e = launch_amax(W, (int64_t)N * K, partial, s);
    if (e != cudaSuccess) return e;
    const dim3 grid(quant_delta_grid(qd_strips(N, K)));
    const ActRows act = {X, X ? M : 0, X ? (M + 127) / 128 * 128 : 0, xcodes, xsf, xsf_swz, g_x};
    if (rcodes)
        return launch_pdl(k_quant_delta<true, true>, grid, dim3(kQDThreads), kQDSmem, s, 1, tw, N, K, H,
                          (const float*)partial, codes, sf, sf_swz, g, rcodes, rsf, delta, err, act);
    return launch_pdl(k_quant_delta<true, false>, grid, dim3(kQDThreads), kQDSmem, s, 1, tw, N, K, H,
                      (const float*)partial, codes, sf, sf_swz, g, (uint8_t*)nullptr, (uint8_t*)nullptr, delta, err,
                      act);
}

// The cluster selection takes more keys than one CTA holds, up to kTkMaxCluster CTAs' worth;
// beyond that the one-CTA kernel reads its keys from global memory in every pass.
int topk_cluster_ctas(int B) {
    if ((size_t)B * 8 <= kSelSmemKeysMax || B > kTkMaxCluster * kTkCtaKeys) return 0;
    return kTkMaxCluster;
}
int topk_cluster_chunk(int B, int C) { return ((B + C - 1) / C + 31) / 32 * 32; }

int topk_launches(int budget) { return budget <= 0 ? 0 : 2; }

cudaError_t launch_topk_select(const double* delta, int B, int budget, int32_t* sel, cudaStream_t s) {
    if (budget <= 0) return cudaSuccess;
    const bool smem_keys = (size_t)B * 8 <= kSelSmemKeysMax;
    const size_t smem = smem_keys ? (size_t)B * 8 : 0;
    static std::atomic<bool> attr_set[64];
    cudaError_t e = once_per_device(attr_set, [] {
        const cudaError_t e1 = cudaFuncSetAttribute(k_topk_large<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    (int)kSelSmemKeysMax + 16 * 1024);
        if (e1 != cudaSuccess) return e1;
        return cudaFuncSetAttribute(k_topk_large<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kSelSmemKeysMax + 16 * 1024);
    });
    if (e != cudaSuccess) return e;
    if (smem_keys) return launch_pdl(k_topk_large<true>, dim3(1), dim3(kSelThreads), smem, s, 1, delta, B, budget, sel);
    const int C = topk_cluster_ctas(B);
    if (C) {
        static std::atomic<bool> attr_c[64];
        e = once_per_device(attr_c, [] {
            return cudaFuncSetAttribute(k_topk_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kTkCtaKeys * (int)sizeof(uint64_t));
        });
        if (e != cudaSuccess) return e;
        const int chunk = topk_cluster_chunk(B, C);
        return launch_pdl_cluster(k_topk_cluster, dim3(C), dim3(kSelThreads), (size_t)chunk * sizeof(uint64_t), s,
                                  dim3(C, 1, 1), delta, B, budget, chunk, sel);
    }
    return launch_pdl(k_topk_large<false>, dim3(1), dim3(kSelThreads), smem, s, 1, delta, B, budget, sel);
}

cudaError_t launch_topk(const double* delta, int B, int budget, int32_t* rank, int32_t* sel, cudaStream_t s) {
    if (budget <= 0) return cudaSuccess;
    cudaError_t e = launch_topk_select(delta, B, budget, sel, s);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_topk_rank_split, dim3((budget + kRankPerCta - 1) / kRankPerCta), dim3(128), 0, s, 1, delta,
                      (const int32_t*)sel, budget, rank);
}

cudaError_t launch_pack(const uint8_t* rcodes, const uint8_t* rsf, int N, int K, const int32_t* sel, int budget,
                        uint8_t* blk_codes, uint8_t* blk_sf, int32_t* blk_kt, int32_t* tile_ptr, uint32_t* bitmap,
                        cudaStream_t s) {
    const int NBr = N / 64;
    const int grid = budget + (NBr + 255) / 256;
    return launch_pdl(k_pack, dim3(grid), dim3(256), 0, s, 1, rcodes, rsf, N, K, sel, budget, blk_codes, blk_sf,
                      blk_kt, tile_ptr, bitmap);
}

cudaError_t launch_pack_w(const uint16_t* W, int N, int K, const float* g_w, const int32_t* sel, int budget,
                          uint8_t* blk_codes, uint8_t* blk_sf, int32_t* blk_kt, int32_t* tile_ptr, uint32_t* bitmap,
                          const double* delta, int32_t* rank, cudaStream_t s) {
    const int NBr = N / 64;
    const int ncsr = (NBr + 127) / 128;
    const int nrank = rank && budget > 0 ? (budget + kRankPerCta - 1) / kRankPerCta : 0;
    return launch_pdl(k_pack_w, dim3(budget + ncsr + nrank), dim3(128), 0, s, 1, W, N, K, g_w, sel, budget, blk_codes,
                      blk_sf, blk_kt, tile_ptr, bitmap, ncsr, delta, nrank ? rank : (int32_t*)nullptr);
}

}  // namespace mq

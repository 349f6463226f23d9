// Block-wise residual allocation (MosaicQuant summary, "Methodology" section 2):
// the Hessian-guided Delta-score of every 64x64 weight block, top-K selection at a
// block budget, and packing of the selected residual blocks for the fused GEMM.
#include "common.cuh"
#include "nvfp4.cuh"
#include "quant.cuh"

namespace mq {

// ------------------------------------------------------------------ Delta-score
// Persistent CTAs (4 warps) walk over the 64x64 blocks (nt, kt); TMA stages each block's
// bf16 tile (64 rows x 128 bytes, 128-byte swizzle) into a ring of shared-memory buffers
// ahead of the arithmetic. Warp q owns group column q (16 K elements); lane r owns block
// rows r and r+32, so the first level of the fixed pairwise row tree (v[i] += v[i+32])
// happens in registers. The remaining levels (+16, +8, +4, +2, +1) run as a butterfly
// over the lanes that at each level also halves the set of columns a lane keeps: the
// adds are exactly the tree's pairs, and at the end lanes 2c and 2c+1 hold column c of
// the group. e and e' are recomputed from W and the tensor scale with the weight
// quantizer's arithmetic, so they are bit-identical to the stored codes.
// tau = fma(e, e, -fp32(e'^2)) (fp32); the column sums are widened to fp64 for
// p_k = H_k c_k and the 64-column tree.
constexpr int kQDStages = 3;
constexpr int kQDTile = 64 * 128;  // bytes of one staged block

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

template <bool kWriteCodes>
__device__ __forceinline__ void quant_delta_block(const uint8_t* tile, int K, const float* __restrict__ H, float g,
                                                  int nt, int kt, uint8_t* __restrict__ codes,
                                                  uint8_t* __restrict__ sf, uint8_t* __restrict__ sf_swz,
                                                  uint8_t* __restrict__ rcodes, uint8_t* __restrict__ rsf,
                                                  double* __restrict__ delta_out, double* pcol, uint32_t* sf_s,
                                                  uint32_t* rsf_s) {
    const int q = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float g6 = __fmul_rn(6.0f, g);
    float a2[2][16];
#pragma unroll
    for (int h = 0; h < 2; ++h) tile_group(tile, lane + 32 * h, q, a2[h]);
    float v[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rl = lane + 32 * h;
        const int64_t row = (int64_t)nt * 64 + rl;
        float deq[16], R[16], rdeq[16];
        uint32_t lo, hi, rlo, rhi;
        const uint32_t sfb = nvfp4_group(a2[h], g, g6, lo, hi, deq);
#pragma unroll
        for (int i = 0; i < 16; ++i) R[i] = __fsub_rn(a2[h][i], deq[i]);
        const uint32_t rsb = nvfp4_group(R, g, g6, rlo, rhi, rdeq);
        if (kWriteCodes) {
            *reinterpret_cast<uint2*>(codes + row * (K / 2) + kt * 32 + q * 8) = make_uint2(lo, hi);
            *reinterpret_cast<uint2*>(rcodes + row * (K / 2) + kt * 32 + q * 8) = make_uint2(rlo, rhi);
            reinterpret_cast<uint8_t*>(sf_s)[rl * 4 + q] = (uint8_t)sfb;
            reinterpret_cast<uint8_t*>(rsf_s)[rl * 4 + q] = (uint8_t)rsb;
        }
        // tau = fma(e, e, -fp32(e'^2)) with e = R, e' = R - deqR; the squares of e' are
        // taken in pairs
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float e0 = R[2 * j], e1 = R[2 * j + 1];
            const float f0 = __fsub_rn(e0, rdeq[2 * j]), f1 = __fsub_rn(e1, rdeq[2 * j + 1]);
            const float2 sq = mul2(make_float2(f0, f1), make_float2(f0, f1));
            const float t0 = __fmaf_rn(e0, e0, -sq.x), t1 = __fmaf_rn(e1, e1, -sq.y);
            v[2 * j] = h ? __fadd_rn(v[2 * j], t0) : t0;
            v[2 * j + 1] = h ? __fadd_rn(v[2 * j + 1], t1) : t1;
        }
    }
    // butterfly: masks 16, 8, 4, 2 keep n = 8, 4, 2, 1 columns; then mask 1 adds pairs
#pragma unroll
    for (int m = 16, n = 8; m >= 2; m >>= 1, n >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int j = 0; j < n; ++j) {
            const float send = upper ? v[j] : v[j + n];
            const float keep = upper ? v[j + n] : v[j];
            v[j] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, m));
        }
    }
    const float colsum = __fadd_rn(v[0], __shfl_xor_sync(0xffffffffu, v[0], 1));
    const int c = (lane >> 1) & 15;
    if ((lane & 1) == 0) pcol[q * 16 + c] = __dmul_rn((double)__ldg(H + kt * 64 + q * 16 + c), (double)colsum);
    __syncthreads();
    if (q == 0) {
        double d = __dadd_rn(pcol[lane], pcol[lane + 32]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d = __dadd_rn(d, __shfl_down_sync(0xffffffffu, d, o));
        if (lane == 0) *delta_out = d;
    }
    if (kWriteCodes && threadIdx.x < 64) {
        const int64_t row = (int64_t)nt * 64 + threadIdx.x;
        const uint32_t wsf = sf_s[threadIdx.x], wr = rsf_s[threadIdx.x];
        if (sf) *reinterpret_cast<uint32_t*>(sf + row * (K / 16) + kt * 4) = wsf;
        *reinterpret_cast<uint32_t*>(rsf + row * (K / 16) + kt * 4) = wr;
        *reinterpret_cast<uint32_t*>(sf_swz + sf_swz_offset(row, (int64_t)kt * 4, K)) = wsf;
    }
}

// A3 (kWriteCodes = false: Delta only, tensor scale read from g_in) and A1 + A3 in one
// pass over W (kWriteCodes = true: codes, scales and Delta, tensor scale from the |W|
// maximum partials). Persistent: CTA c handles blocks c, c + gridDim.x, ...
template <bool kWriteCodes>
__global__ void __launch_bounds__(128) k_quant_delta(const __grid_constant__ CUtensorMap tmap_w, int N, int K,
                                                     const float* __restrict__ H, const float* __restrict__ g_in,
                                                     uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                     uint8_t* __restrict__ sf_swz, float* __restrict__ g_out,
                                                     uint8_t* __restrict__ rcodes, uint8_t* __restrict__ rsf,
                                                     double* __restrict__ delta, int* __restrict__ err) {
    extern __shared__ uint8_t qd_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qd_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(tiles + kQDStages * kQDTile);
    __shared__ double pcol[64];
    __shared__ uint32_t sf_s[64], rsf_s[64];
    griddep_wait();
    griddep_launch();
    const float g = kWriteCodes ? tensor_scale(g_in) : __ldg(g_in);
    if (kWriteCodes && blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
    const int KB = K / 64, NB = (N / 64) * KB;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQDStages; ++s) mbar_init(&full[s], 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmap_w);
    }
    __syncthreads();
    auto issue = [&](int i) {  // block number i of this CTA into stage i % kQDStages
        const int b = blockIdx.x + i * gridDim.x;
        if (b < NB) {
            const int s = i % kQDStages;
            mbar_arrive_expect_tx(&full[s], kQDTile);
            tma_load_2d_u16(tiles + s * kQDTile, &tmap_w, &full[s], (b % KB) * 64, (b / KB) * 64);
        }
    };
    if (threadIdx.x == 0)
        for (int i = 0; i < kQDStages; ++i) issue(i);
    bool ok = true;
    for (int i = 0;; ++i) {
        const int b = blockIdx.x + i * gridDim.x;
        if (b >= NB) break;
        const int s = i % kQDStages;
        if (ok) ok = mbar_wait_err(&full[s], (i / kQDStages) & 1, err);
        if (ok)
            quant_delta_block<kWriteCodes>(tiles + s * kQDTile, K, H, g, b / KB, b % KB, codes, sf, sf_swz, rcodes,
                                           rsf, delta + b, pcol, sf_s, rsf_s);
        __syncthreads();  // stage s and the block's shared scratch are free again
        // every copy issued here is waited for by a later iteration of this loop
        if (threadIdx.x == 0 && ok) issue(i + kQDStages);
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

// Single-CTA radix select of the budget-th largest key (8 digits of 8 bits, most
// significant first; keys held in shared memory when they fit), then a stable
// compaction in block order: every key above the threshold plus the lowest-index keys
// equal to it, which writes sel ascending. With kRank the same CTA also writes rank by
// counting: position of selected i = #{j : key_j > key_i} + #{j < i : key_j == key_i}.
constexpr int kSelThreads = 1024;
constexpr int kRankInCtaMax = 1024;        // budgets up to this are ranked in the CTA
constexpr size_t kSelSmemKeysMax = 160 * 1024;

template <bool kSmemKeys, bool kRank>
__global__ void __launch_bounds__(kSelThreads) k_topk(const double* __restrict__ delta, int B, int budget,
                                                      int32_t* __restrict__ sel, int32_t* __restrict__ rank) {
    griddep_wait();
    griddep_launch();
    extern __shared__ __align__(16) uint64_t dyn[];
    uint64_t* keys = dyn;                                   // [B] when kSmemKeys
    uint64_t* selkey = dyn + (kSmemKeys ? B : 0);           // [budget] when kRank
    int32_t* selidx = reinterpret_cast<int32_t*>(selkey + (kRank ? budget : 0));
    __shared__ unsigned hist[256];
    __shared__ uint64_t s_prefix, s_mask;
    __shared__ int s_need;
    __shared__ int scratch[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (kSmemKeys)
        for (int i = tid; i < B; i += kSelThreads) keys[i] = order_key(delta[i]);
    if (tid == 0) { s_prefix = 0; s_mask = 0; s_need = budget; }
    __syncthreads();
    auto key_of = [&](int i) -> uint64_t { return kSmemKeys ? keys[i] : order_key(delta[i]); };
#pragma unroll 1
    for (int shift = 56; shift >= 0; shift -= 8) {
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        const uint64_t prefix = s_prefix, mask = s_mask;
        // warp-aggregated histogram: lanes with the same digit add once (the keys share
        // their leading digits, so per-lane atomics would all hit one bin)
        for (int i0 = tid - lane; i0 < B; i0 += kSelThreads) {
            const int i = i0 + lane;
            unsigned digit = 256u;  // not counted
            if (i < B) {
                const uint64_t key = key_of(i);
                if ((key & mask) == prefix) digit = (unsigned)(key >> shift) & 255u;
            }
            const unsigned peers = __match_any_sync(0xffffffffu, digit);
            if (digit < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (unsigned)__popc(peers));
        }
        __syncthreads();
        if (warp == 0) {
            // lane l scans bins 255-8l down to 248-8l; find the bin where the count of
            // keys from the top reaches `need`
            unsigned cnt[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { cnt[j] = hist[255 - 8 * lane - j]; tot += cnt[j]; }
            unsigned incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int need = s_need;
            const unsigned hit = __ballot_sync(0xffffffffu, incl >= (unsigned)need);
            const int first = __ffs(hit) - 1;
            if (lane == first) {
                unsigned cum = incl - tot;
                int digit = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (cum + cnt[j] >= (unsigned)need) { digit = 255 - 8 * lane - j; break; }
                    cum += cnt[j];
                }
                s_need = need - (int)cum;
                s_prefix = prefix | ((uint64_t)digit << shift);
                s_mask = mask | ((uint64_t)255 << shift);
            }
        }
        __syncthreads();
    }
    const uint64_t T = s_prefix;
    const int need_eq = s_need;  // how many keys equal to T are taken (lowest b first)
    const int chunk = (B + kSelThreads - 1) / kSelThreads;
    const int lo = min(B, tid * chunk), hi = min(B, lo + chunk);
    int gt = 0, eq = 0;
    for (int i = lo; i < hi; ++i) {
        const uint64_t key = key_of(i);
        gt += key > T;
        eq += key == T;
    }
    int total;
    const int eq_before = block_exclusive_sum<kSelThreads>(eq, scratch, total);
    const int eq_take = max(0, min(eq, need_eq - eq_before));
    int out = block_exclusive_sum<kSelThreads>(gt + eq_take, scratch, total);
    int eq_seen = eq_before;
    for (int i = lo; i < hi; ++i) {
        const uint64_t key = key_of(i);
        bool take = key > T;
        if (key == T) take = eq_seen++ < need_eq;
        if (take) {
            sel[out] = i;
            if (kRank) { selkey[out] = key; selidx[out] = i; }
            ++out;
        }
    }
    if (kRank) {
        // position of selected i, counted in `parts` slices of j by different threads
        __shared__ int pos_s[kRankInCtaMax];
        for (int i = tid; i < budget; i += kSelThreads) pos_s[i] = 0;
        __syncthreads();
        const int parts = max(1, kSelThreads / budget);
        const int span = (budget + parts - 1) / parts;
        for (int w = tid; w < budget * parts; w += kSelThreads) {
            const int i = w / parts, part = w % parts;
            const uint64_t mine = selkey[i];
            const int j0 = part * span, j1 = min(budget, j0 + span);
            int pos = 0;
            for (int j = j0; j < j1; ++j) {
                const uint64_t kj = selkey[j];
                pos += (kj > mine) | ((kj == mine) & (j < i));
            }
            atomicAdd(&pos_s[i], pos);
        }
        __syncthreads();
        for (int i = tid; i < budget; i += kSelThreads) rank[pos_s[i]] = selidx[i];
    }
}

// Top-K for budgets up to kSmallBudget, one CTA:
//  1. keys (order-preserving 64-bit images of Delta) and their common leading bits;
//  2. 8-bit radix passes below the common prefix until at most kCandMax keys share the
//     bucket that holds the budget-th largest key (warp-uniform digits add once);
//  3. the keys of higher buckets (all selected) and the candidates of that bucket go
//     into one list, sorted by (key descending, block index ascending), a strict total
//     order: its first `budget` entries are rank; sel is the same set in ascending block
//     index, from a bitmap scan.
// If the keys tie beyond kCandMax candidates (the bucket is resolved to a single key
// value), the selected set is compacted in block order instead (every key above the
// value, then the lowest-index keys equal to it) and then sorted for rank.
constexpr int kSmallBudget = 1024;
constexpr int kCandMax = 512;
constexpr int kSortCap = 2048;  // budget + candidates, a power of two

__device__ __forceinline__ bool before(uint64_t ka, int ia, uint64_t kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// Bitonic sort of n2 (power of two, <= 2 * blockDim.x) (key, idx) pairs in shared memory
// by (key descending, idx ascending). Pair p belongs to thread p; a warp's pairs cover 64
// consecutive elements for strides below 64, which then need only __syncwarp.
__device__ __forceinline__ void block_sort_desc(uint64_t* key, int32_t* idx, int n2) {
    const int p = threadIdx.x;
    const bool act = p < (n2 >> 1);
    for (int k = 2, lk = 1; k <= n2; k <<= 1, ++lk) {
        for (int j = k >> 1, lj = lk - 1; j > 0; j >>= 1, --lj) {
            if (act) {
                const int i = ((p >> lj) << (lj + 1)) | (p & (j - 1)), q = i + j;
                const bool desc = (i & k) == 0;
                const uint64_t ki = key[i], kq = key[q];
                const int ii = idx[i], iq = idx[q];
                if (before(kq, iq, ki, ii) == desc) {
                    key[i] = kq;
                    key[q] = ki;
                    idx[i] = iq;
                    idx[q] = ii;
                }
            }
            const int jn = j > 1 ? (j >> 1) : k;  // the next stage's stride
            if (j >= 64 || jn >= 64) __syncthreads();
            else __syncwarp();
        }
    }
}

__device__ __forceinline__ uint64_t warp_and64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v &= __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ uint64_t warp_or64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <bool kSmemKeys>
__global__ void __launch_bounds__(kSelThreads) k_topk_small(const double* __restrict__ delta, int B, int budget,
                                                            int32_t* __restrict__ rank, int32_t* __restrict__ sel) {
    extern __shared__ __align__(16) uint64_t dyn[];
    uint64_t* keys = dyn;                                         // [B] when kSmemKeys
    uint64_t* skey = dyn + (kSmemKeys ? B : 0);                   // [kSortCap]
    int32_t* sidx = reinterpret_cast<int32_t*>(skey + kSortCap);  // [kSortCap]
    uint32_t* bits = reinterpret_cast<uint32_t*>(sidx + kSortCap); // [ceil(B / 32)]
    __shared__ unsigned hist[256];
    __shared__ uint64_t s_and[32], s_or[32];
    __shared__ uint64_t s_prefix;
    __shared__ int s_pos, s_need, s_cand, s_nsel;
    __shared__ int scratch[32];
    griddep_wait();  // Delta comes from the previous kernel
    griddep_launch();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nw = (B + 31) / 32;
    auto key_of = [&](int i) -> uint64_t { return kSmemKeys ? keys[i] : order_key(delta[i]); };

    uint64_t a = ~0ull, o = 0ull;
    for (int i = tid; i < B; i += kSelThreads) {
        const uint64_t k = order_key(delta[i]);
        if (kSmemKeys) keys[i] = k;
        a &= k;
        o |= k;
    }
    for (int w = tid; w < nw; w += kSelThreads) bits[w] = 0u;
    a = warp_and64(a);
    o = warp_or64(o);
    if (lane == 0) { s_and[warp] = a; s_or[warp] = o; }
    __syncthreads();
    if (warp == 0) {
        a = s_and[lane];
        o = s_or[lane];
        a = warp_and64(a);
        o = warp_or64(o);
        if (lane == 0) {
            const int cp = (a ^ o) ? __clzll((long long)(a ^ o)) : 64;  // common leading bits
            s_pos = 64 - cp;
            s_prefix = cp ? (a & (~0ull << (64 - cp))) : 0ull;
            s_need = budget;
            s_cand = B;
            s_nsel = 0;
        }
    }
    __syncthreads();
    // radix passes below the common prefix
    while (s_pos > 0 && s_cand > kCandMax) {
        const int pos = s_pos, w = pos < 8 ? pos : 8, shift = pos - w;
        const uint64_t prefix = s_prefix, hi = pos >= 64 ? 0ull : (~0ull << pos);
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int i0 = tid - lane; i0 < B; i0 += kSelThreads) {
            const int i = i0 + lane;
            unsigned digit = 256u;
            if (i < B) {
                const uint64_t k = key_of(i);
                if ((k & hi) == prefix) digit = (unsigned)(k >> shift) & ((1u << w) - 1u);
            }
            const bool uniform = __all_sync(0xffffffffu, digit == __shfl_sync(0xffffffffu, digit, 0));
            if (uniform) {
                if (lane == 0 && digit < 256u) atomicAdd(&hist[digit], 32u);
            } else if (digit < 256u) {
                atomicAdd(&hist[digit], 1u);
            }
        }
        __syncthreads();
        if (warp == 0) {
            // bins from the top: lane l holds bins 255-8l .. 248-8l
            unsigned cnt[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { cnt[j] = hist[255 - 8 * lane - j]; tot += cnt[j]; }
            unsigned incl = tot;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const unsigned y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += y;
            }
            const int need = s_need;
            const unsigned hit = __ballot_sync(0xffffffffu, incl >= (unsigned)need);
            const int first = __ffs(hit) - 1;
            if (lane == first) {
                unsigned cum = incl - tot;
                int digit = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (cum + cnt[j] >= (unsigned)need) {
                        digit = 255 - 8 * lane - j;
                        s_cand = (int)cnt[j];
                        break;
                    }
                    cum += cnt[j];
                }
                s_need = need - (int)cum;
                s_prefix = prefix | ((uint64_t)digit << shift);
                s_pos = shift;
            }
        }
        __syncthreads();
    }
    const int pos = s_pos, need = s_need;
    const uint64_t prefix = s_prefix, hi = pos >= 64 ? 0ull : (~0ull << pos);
    if (s_cand <= kCandMax) {
        // every key above the bucket plus the bucket's candidates, then one sort
        for (int i = tid; i < B; i += kSelThreads) {
            const uint64_t k = key_of(i);
            const uint64_t kh = k & hi;
            if (kh >= prefix) {
                const int slot = atomicAdd(&s_nsel, 1);
                skey[slot] = k;
                sidx[slot] = i;
            }
        }
        __syncthreads();
        const int nsel = s_nsel;
        int n2 = 2;
        while (n2 < nsel) n2 <<= 1;
        for (int e = nsel + tid; e < n2; e += kSelThreads) { skey[e] = 0ull; sidx[e] = 0x7FFFFFFF - e; }
        __syncthreads();
        block_sort_desc(skey, sidx, n2);
    } else {
        // the bucket is a single key value T shared by more than kCandMax keys: keys above
        // T and the lowest-index `need` keys equal to T, compacted in block order
        const uint64_t T = prefix;
        const int chunk = (B + kSelThreads - 1) / kSelThreads;
        const int lo = min(B, tid * chunk), hi2 = min(B, lo + chunk);
        int gt = 0, eq = 0;
        for (int i = lo; i < hi2; ++i) {
            const uint64_t k = key_of(i);
            gt += k > T;
            eq += k == T;
        }
        int total;
        const int eq_before = block_exclusive_sum<kSelThreads>(eq, scratch, total);
        const int eq_take = max(0, min(eq, need - eq_before));
        int out = block_exclusive_sum<kSelThreads>(gt + eq_take, scratch, total);
        int eq_seen = eq_before;
        for (int i = lo; i < hi2; ++i) {
            const uint64_t k = key_of(i);
            bool take = k > T;
            if (k == T) take = eq_seen++ < need;
            if (take) { skey[out] = k; sidx[out] = i; ++out; }
        }
        __syncthreads();
        int n2 = 2;
        while (n2 < budget) n2 <<= 1;
        for (int e = budget + tid; e < n2; e += kSelThreads) { skey[e] = 0ull; sidx[e] = 0x7FFFFFFF - e; }
        __syncthreads();
        block_sort_desc(skey, sidx, n2);
    }
    for (int e = tid; e < budget; e += kSelThreads) {
        rank[e] = sidx[e];
        atomicOr(&bits[sidx[e] >> 5], 1u << (sidx[e] & 31));
    }
    __syncthreads();
    // sel: the set bits in index order (each thread scans a run of bitmap words)
    const int per = (nw + kSelThreads - 1) / kSelThreads;
    const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bits[w]);
    int total;
    int out = block_exclusive_sum<kSelThreads>(cnt, scratch, total);
    for (int w = w0; w < w1; ++w) {
        uint32_t b = bits[w];
        while (b) {
            const int t = __ffs(b) - 1;
            b &= b - 1;
            sel[out++] = w * 32 + t;
        }
    }
}

// rank: position of selected block i = #{j : key_j > key_i} + #{j < i : key_j == key_i}
// (sel is ascending, so a lower list index is a lower block index).
__global__ void __launch_bounds__(256) k_topk_rank(const double* __restrict__ delta, const int32_t* __restrict__ sel,
                                                   int budget, int32_t* __restrict__ rank) {
    griddep_wait();
    griddep_launch();
    __shared__ uint64_t keys[2048];
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const uint64_t mine = i < budget ? order_key(delta[sel[i]]) : 0;
    int pos = 0;
    for (int base = 0; base < budget; base += 2048) {
        const int n = min(2048, budget - base);
        __syncthreads();
        for (int j = threadIdx.x; j < n; j += blockDim.x) keys[j] = order_key(delta[sel[base + j]]);
        __syncthreads();
        if (i < budget) {
            for (int j = 0; j < n; ++j) {
                const uint64_t kj = keys[j];
                pos += (kj > mine) | ((kj == mine) & (base + j < i));
            }
        }
    }
    if (i < budget) rank[pos] = sel[i];
}

// ------------------------------------------------------------------ pack
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
    const int KB = K / 64, NBr = N / 64, KW = (KB + 31) / 32;
    if ((int)blockIdx.x < budget) {
        const int i = blockIdx.x;
        const int b = __ldg(sel + i), nt = b / KB, kt = b % KB;
        const int t = threadIdx.x;
        {   // codes: row r, bytes 8*c8 .. 8*c8+7 of the block row
            const int r = t >> 2, c8 = t & 3, j = 8 * c8;
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(rcodes + (int64_t)(nt * 64 + r) * (K / 2) + kt * 32 + j));
            const int off = (r >> 3) * 256 + (j >> 4) * 128 + (r & 7) * 16 + (j & 15);
            *reinterpret_cast<uint2*>(blk_codes + (int64_t)i * 2048 + off) = v;
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
    const int nt = (blockIdx.x - budget) * blockDim.x + threadIdx.x;
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

// ------------------------------------------------------------------ launchers
static int quant_delta_grid(int NB) {
    static int per_sm = 0;
    if (!per_sm) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quant_delta<true>, 128,
                                                          kQDStages * kQDTile + 1024 + 64) != cudaSuccess ||
            per_sm < 1)
            per_sm = 4;
    }
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = per_sm * sms;
    return NB < grid ? NB : grid;
}

static const size_t kQDSmem = kQDStages * kQDTile + 1024 + 64;

cudaError_t launch_delta(const CUtensorMap& tw, int N, int K, const float* H, const float* g, double* delta,
                         int* err, cudaStream_t s) {
    const int NB = (N / 64) * (K / 64);
    return launch_pdl(k_quant_delta<false>, dim3(quant_delta_grid(NB)), dim3(128), kQDSmem, s, 1, tw, N, K, H, g,
                      (uint8_t*)nullptr, (uint8_t*)nullptr, (uint8_t*)nullptr, (float*)nullptr, (uint8_t*)nullptr,
                      (uint8_t*)nullptr, delta, err);
}

cudaError_t launch_quant_delta(const uint16_t* W, const CUtensorMap& tw, int N, int K, const float* H,
                               uint8_t* codes, uint8_t* sf, uint8_t* sf_swz, float* g, uint8_t* rcodes, uint8_t* rsf,
                               double* delta, float* partial, int* err, cudaStream_t s) {
    cudaError_t e = launch_amax(W, (int64_t)N * K, partial, s);
    if (e != cudaSuccess) return e;
    const int NB = (N / 64) * (K / 64);
    return launch_pdl(k_quant_delta<true>, dim3(quant_delta_grid(NB)), dim3(128), kQDSmem, s, 1, tw, N, K, H,
                      (const float*)partial, codes, sf, sf_swz, g, rcodes, rsf, delta, err);
}

cudaError_t launch_topk(const double* delta, int B, int budget, int32_t* rank, int32_t* sel, cudaStream_t s) {
    if (budget <= 0) return cudaSuccess;
    if (budget <= kSmallBudget) {
        const size_t tail = (size_t)kSortCap * 12 + (size_t)((B + 31) / 32) * 4;
        const bool smem_keys = (size_t)B * 8 + tail <= kSelSmemKeysMax;
        const size_t smem = (smem_keys ? (size_t)B * 8 : 0) + tail;
        static bool attr[2] = {false, false};
        auto go = [&](auto kern, int which) -> cudaError_t {
            if (!attr[which]) {
                cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)kSelSmemKeysMax + 16 * 1024);
                if (e != cudaSuccess) return e;
                attr[which] = true;
            }
            return launch_pdl(kern, dim3(1), dim3(kSelThreads), smem, s, 1, delta, B, budget, rank, sel);
        };
        return smem_keys ? go(k_topk_small<true>, 0) : go(k_topk_small<false>, 1);
    }
    // larger budgets: radix select and compaction, then a separate counting rank kernel
    const bool smem_keys = (size_t)B * 8 <= kSelSmemKeysMax;
    const size_t smem = smem_keys ? (size_t)B * 8 : 0;
    static bool attr2[2] = {false, false};
    auto go2 = [&](auto kern, int which) -> cudaError_t {
        if (!attr2[which]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kSelSmemKeysMax + 16 * 1024);
            if (e != cudaSuccess) return e;
            attr2[which] = true;
        }
        return launch_pdl(kern, dim3(1), dim3(kSelThreads), smem, s, 1, delta, B, budget, sel, rank);
    };
    cudaError_t e = smem_keys ? go2(k_topk<true, false>, 0) : go2(k_topk<false, false>, 1);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_topk_rank, dim3((budget + 255) / 256), dim3(256), 0, s, 1, delta, (const int32_t*)sel, budget,
                      rank);
}

cudaError_t launch_pack(const uint8_t* rcodes, const uint8_t* rsf, int N, int K, const int32_t* sel, int budget,
                        uint8_t* blk_codes, uint8_t* blk_sf, int32_t* blk_kt, int32_t* tile_ptr, uint32_t* bitmap,
                        cudaStream_t s) {
    const int NBr = N / 64;
    const int grid = budget + (NBr + 255) / 256;
    return launch_pdl(k_pack, dim3(grid), dim3(256), 0, s, 1, rcodes, rsf, N, K, sel, budget, blk_codes, blk_sf,
                      blk_kt, tile_ptr, bitmap);
}

}  // namespace mq

// Block-wise residual allocation (MosaicQuant summary, "Methodology" section 2):
// the Hessian-guided Delta-score of every 64x64 weight block, top-K selection at a
// block budget, and packing of the selected residual blocks for the fused GEMM.
#include "common.cuh"
#include "nvfp4.cuh"

namespace mq {

// ------------------------------------------------------------------ Delta-score
// One CTA per block (nt, kt), thread (r = tid/4, q = tid%4) owns one 16-group of the
// block. e and e' are recomputed from W and the tensor scale exactly as the weight
// quantizer computes them, so no codes are re-read. The reductions follow the fixed
// pairwise tree v[i] += v[i+32], +16, +8, +4, +2, +1 (rows first, then columns).
constexpr int kTauStride = 65;  // fp64 words per smem row (pad: conflict-free columns)

__global__ void __launch_bounds__(256) k_delta(const uint16_t* __restrict__ W, int N, int K,
                                               const float* __restrict__ H, const float* __restrict__ gptr,
                                               double* __restrict__ delta) {
    __shared__ double tau[64 * kTauStride];
    __shared__ double p[64];
    const int KB = K / 64;
    const int b = blockIdx.x;
    const int nt = b / KB, kt = b % KB;
    const int r = threadIdx.x >> 2, q = threadIdx.x & 3;
    const float g = __ldg(gptr);
    const float g6 = __fmul_rn(6.0f, g);
    {
        float a[16], deq[16], R[16], rdeq[16];
        const uint4* src = reinterpret_cast<const uint4*>(W + (int64_t)(nt * 64 + r) * K + kt * 64 + q * 16);
        const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
            a[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
        }
        uint32_t lo, hi;
        nvfp4_group(a, g, g6, lo, hi, deq);
#pragma unroll
        for (int i = 0; i < 16; ++i) R[i] = __fsub_rn(a[i], deq[i]);
        nvfp4_group(R, g, g6, lo, hi, rdeq);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const double e = (double)R[i];
            const double e2 = (double)__fsub_rn(R[i], rdeq[i]);
            tau[r * kTauStride + q * 16 + i] = __dsub_rn(__dmul_rn(e, e), __dmul_rn(e2, e2));
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll 1
    for (int c = warp * 8; c < warp * 8 + 8; ++c) {
        double v = __dadd_rn(tau[lane * kTauStride + c], tau[(lane + 32) * kTauStride + c]);
#pragma unroll
        for (int h = 16; h > 0; h >>= 1) v = __dadd_rn(v, __shfl_down_sync(0xffffffffu, v, h));
        if (lane == 0) p[c] = __dmul_rn((double)__ldg(H + kt * 64 + c), v);
    }
    __syncthreads();
    if (warp == 0) {
        double v = __dadd_rn(p[lane], p[lane + 32]);
#pragma unroll
        for (int h = 16; h > 0; h >>= 1) v = __dadd_rn(v, __shfl_down_sync(0xffffffffu, v, h));
        if (lane == 0) delta[b] = v;
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
// significant first), then a stable compaction in block order: every key above the
// threshold plus the lowest-index keys equal to it. Writes sel ascending.
constexpr int kSelThreads = 1024;

__global__ void __launch_bounds__(kSelThreads) k_topk_select(const double* __restrict__ delta, int B, int budget,
                                                             int32_t* __restrict__ sel) {
    __shared__ unsigned hist[256];
    __shared__ uint64_t s_prefix, s_mask;
    __shared__ int s_need;
    __shared__ int scratch[32];
    if (threadIdx.x == 0) { s_prefix = 0; s_mask = 0; s_need = budget; }
    __syncthreads();
#pragma unroll 1
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        const uint64_t prefix = s_prefix, mask = s_mask;
        for (int i = threadIdx.x; i < B; i += kSelThreads) {
            const uint64_t key = order_key(delta[i]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int need = s_need;
            unsigned cum = 0;
            int digit = 0;
            for (int d = 255; d >= 0; --d) {
                if (cum + hist[d] >= (unsigned)need) { digit = d; break; }
                cum += hist[d];
            }
            s_need = need - (int)cum;
            s_prefix = prefix | ((uint64_t)digit << shift);
            s_mask = mask | ((uint64_t)255 << shift);
        }
        __syncthreads();
    }
    const uint64_t T = s_prefix;
    const int need_eq = s_need;  // how many keys equal to T are taken (lowest b first)
    const int chunk = (B + kSelThreads - 1) / kSelThreads;
    const int lo = min(B, (int)threadIdx.x * chunk), hi = min(B, lo + chunk);
    int gt = 0, eq = 0;
    for (int i = lo; i < hi; ++i) {
        const uint64_t key = order_key(delta[i]);
        gt += key > T;
        eq += key == T;
    }
    int total;
    const int eq_before = block_exclusive_sum<kSelThreads>(eq, scratch, total);
    const int eq_take = max(0, min(eq, need_eq - eq_before));
    int out = block_exclusive_sum<kSelThreads>(gt + eq_take, scratch, total);
    int eq_seen = eq_before;
    for (int i = lo; i < hi; ++i) {
        const uint64_t key = order_key(delta[i]);
        bool take = key > T;
        if (key == T) take = eq_seen++ < need_eq;
        if (take) sel[out++] = i;
    }
}

// rank: position of selected block i = #{j : key_j > key_i} + #{j < i : key_j == key_i}
// (sel is ascending, so a lower list index is a lower block index).
__global__ void __launch_bounds__(256) k_topk_rank(const double* __restrict__ delta, const int32_t* __restrict__ sel,
                                                   int budget, int32_t* __restrict__ rank) {
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
cudaError_t launch_delta(const uint16_t* W, int N, int K, const float* H, const float* g, double* delta,
                         cudaStream_t s) {
    const int B = (N / 64) * (K / 64);
    k_delta<<<B, 256, 0, s>>>(W, N, K, H, g, delta);
    return cudaGetLastError();
}

cudaError_t launch_topk(const double* delta, int B, int budget, int32_t* rank, int32_t* sel, cudaStream_t s) {
    if (budget <= 0) return cudaSuccess;
    k_topk_select<<<1, kSelThreads, 0, s>>>(delta, B, budget, sel);
    k_topk_rank<<<(budget + 255) / 256, 256, 0, s>>>(delta, sel, budget, rank);
    return cudaGetLastError();
}

cudaError_t launch_pack(const uint8_t* rcodes, const uint8_t* rsf, int N, int K, const int32_t* sel, int budget,
                        uint8_t* blk_codes, uint8_t* blk_sf, int32_t* blk_kt, int32_t* tile_ptr, uint32_t* bitmap,
                        cudaStream_t s) {
    const int NBr = N / 64;
    const int grid = budget + (NBr + 255) / 256;
    k_pack<<<grid, 256, 0, s>>>(rcodes, rsf, N, K, sel, budget, blk_codes, blk_sf, blk_kt, tile_ptr, bitmap);
    return cudaGetLastError();
}

}  // namespace mq

// Types and entry points of the fused GEMM shared by the kernels and the host API.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "mosaic.h"

namespace mq {

struct GemmParams {
    const uint8_t* w_sf;     // tiled scales of W
    const uint8_t* x_sf;     // tiled scales of X
    const float* g_w;        // [1]
    const float* g_x;        // [M]
    const uint8_t* blk_codes;
    const uint8_t* blk_sf;
    const int32_t* tile_ptr;
    const uint32_t* bitmap;
    uint16_t* Y;
    float* partial;          // split-K partials [splits][tiles_m * BN][N]
    int* counters;           // [tiles_m * tiles_n], zero between calls
    int M, N, K;
    int splits, iters_per_split;
    int mode;                // 0 fused, 1 base only, 2 residual only
    int has_resid;
    int nblk;                // packed residual blocks (when has_resid)
    int cluster;             // split-K reduced through the cluster's shared memory
    int prefetch;            // W and X were complete before this kernel could start, so the
                             // decode kernel may load them before waiting for its predecessor
    int w_ready;             // W, its scales and the packed residual were complete before this
                             // kernel could start (X may not be): W may be loaded before the wait
    const uint16_t* x_bf16;  // decode kernel: bf16 X [M][K] quantized inside the kernel
                             // (x_sf and g_x unused), or null
    float* gx_out;           // with x_bf16: per-token scales written here if not null
    // stream-K decode kernel: `units` = tiles x (K / 256) work units, CTA c takes units
    // [c * units / grid, (c + 1) * units / grid); tile t = n_tile * tiles_m + m_tile
    int units, tiles_m, tiles_n;
    unsigned long long wait_ns;  // stream-K kernel: wall-clock limit of every pipeline wait
    int skip_unit;               // test hook: CTA 0 does not request this unit's W (-1: none)
};

// Stream-K decode kernel plan: token tile BN (the MMA's N side), tiles_n x tiles_m
// output tiles of 128 weight rows x BN tokens, `grid` persistent CTAs sharing the
// tiles x (K / 256) units equally; `ws` workspace bytes (0 when no tile is split).
struct StreamKPlan {
    int BN, tiles_m, tiles_n, units, grid;
    size_t ws;
    size_t slots_bytes;  // partial slots before the tile counters
};

StreamKPlan plan_streamk(int M, int N, int K);
// Small decode problems (M <= 32, at most half as many 128-row tiles as SMs, short K
// ranges): the cluster split S (>= 1) of each tile's K range, or 0 for the stream-K kernel.
int plan_small(int M, int N, int K);
cudaError_t launch_gemm_small(const CUtensorMap& tw, const CUtensorMap& tx, GemmParams p, int S, cudaStream_t s);
cudaError_t launch_gemm_streamk(const CUtensorMap& tw, const CUtensorMap& tx, GemmParams p, const StreamKPlan& d,
                                cudaStream_t s);

// Decode kernel tiling: token tile BN, grid tiles_n x splits x tiles_m, `iters`
// K stages (256 elements each) per split.
struct DecodePlan {
    int BN, tiles_m, tiles_n, splits, iters;
    bool cluster;  // splits reduced in a (1, splits, 1) cluster, no workspace
};

DecodePlan plan_decode(int M, int N, int K);
size_t decode_workspace_bytes(int M, int N, int K);
cudaError_t launch_gemm_decode(const CUtensorMap& tw, const CUtensorMap& tx, GemmParams p, const DecodePlan& d,
                               cudaStream_t s);
// Large-M kernel on CTA pairs: W and X code maps with 128-row boxes, u32 maps over the
// tiled scales (128 x 4 boxes: four 512-byte chunks) and over the packed residual (codes
// as rows of 1 KB, scales as rows of 512 B).
cudaError_t launch_gemm_prefill2(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& twsf,
                                 const CUtensorMap& txsf, const CUtensorMap& trc, const CUtensorMap& trsf,
                                 const GemmParams& p, cudaStream_t s);
cudaError_t read_clear_error(int* value);

// The fused GEMM's host side (api.cu), shared by mq_gemm and mq_gemm_noalloc.
mq_status gemm_dispatch(const mq_nvfp4_mat* xq, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y,
                        int M, int N, int K, unsigned flags, void* ws, size_t ws_bytes, bool prefetch,
                        bool clear_counters, mq_stream stream);
cudaError_t error_word(int** ptr);

}  // namespace mq

// Host side of libmosaic: argument validation, TMA descriptors and kernel dispatch
// behind the C ABI declared in mosaic.h.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "gemm.cuh"
#include "mosaic_test.h"

namespace mq {

// launchers (quant.cu, select.cu, gemm.cu)
int amax_grid(int64_t n8);
cudaError_t launch_quant_weight(const uint16_t* W, int N, int K, uint8_t* codes, uint8_t* sf, uint8_t* sf_swz,
                                float* g, uint8_t* rcodes, uint8_t* rsf, float* partial, cudaStream_t s);
cudaError_t launch_quant_act(const uint16_t* X, int M, int K, uint8_t* codes, uint8_t* sf, uint8_t* sf_swz,
                             float* g, bool early, cudaStream_t s);
cudaError_t launch_hessian(const uint16_t* X, int T, int K, float* H, cudaStream_t s);
int hessian_max_tokens();
cudaError_t launch_delta(const CUtensorMap& tw, int N, int K, const float* H, const float* g, double* delta,
                         int* err, cudaStream_t s);
cudaError_t launch_quant_delta(const uint16_t* W, const CUtensorMap& tw, int N, int K, const float* H,
                               uint8_t* codes, uint8_t* sf, uint8_t* sf_swz, float* g, uint8_t* rcodes, uint8_t* rsf,
                               double* delta, float* partial, int* err, cudaStream_t s, const uint16_t* X, int M,
                               uint8_t* xcodes, uint8_t* xsf, uint8_t* xsf_swz, float* g_x);
bool quant_delta_takes_act(int K);
cudaError_t launch_topk(const double* delta, int B, int budget, int32_t* rank, int32_t* sel, cudaStream_t s);
int topk_launches(int budget);
cudaError_t launch_pack(const uint8_t* rcodes, const uint8_t* rsf, int N, int K, const int32_t* sel, int budget,
                        uint8_t* blk_codes, uint8_t* blk_sf, int32_t* blk_kt, int32_t* tile_ptr, uint32_t* bitmap,
                        cudaStream_t s);
cudaError_t launch_pack_w(const uint16_t* W, int N, int K, const float* g_w, const int32_t* sel, int budget,
                          uint8_t* blk_codes, uint8_t* blk_sf, int32_t* blk_kt, int32_t* tile_ptr, uint32_t* bitmap,
                          const double* delta, int32_t* rank, cudaStream_t s);
cudaError_t launch_topk_select(const double* delta, int B, int budget, int32_t* sel, cudaStream_t s);
cudaError_t launch_smooth_scales(const uint16_t* Xcal, int T, const uint16_t* W, int N, int K, float* s,
                                 cudaStream_t st);
cudaError_t launch_smooth_apply(const uint16_t* A, int rows, int K, const float* s, int invert, uint16_t* out,
                                cudaStream_t st);

}  // namespace mq

using namespace mq;

static std::atomic<uint64_t> g_launches{0};

// Test hook (mq_test_arm_wait_fault): the next decode GEMM launch skips one unit's W copies
// in CTA 0 and gives up each wait after g_fault_ns.
static std::atomic<int> g_fault_unit{-1};
static std::atomic<unsigned long long> g_fault_ns{0};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D byte tensor [rows][row_bytes] (row-major), 128-byte swizzled boxes of
// box_bytes x box_rows; rows outside the tensor read as zero.
static bool make_tmap_bytes(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                            uint32_t box_bytes, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_bytes, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// u32 matrix [rows][row_u32] (row-major, no swizzle) in boxes of box_u32 x box_rows.
static bool make_tmap_u32(CUtensorMap* map, const void* base, uint64_t row_u32, uint64_t rows, uint32_t box_u32,
                          uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {row_u32, rows};
    cuuint64_t strides[1] = {row_u32 * 4};
    cuuint32_t box[2] = {box_u32, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 matrix [rows][cols] in 64-column x 128-row boxes with the 128-byte swizzle (two
// stacked Delta blocks); rows outside the matrix read as zero.
static bool make_tmap_bf16_blocks(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Device address of the library's error word (looked up once per device).
static int* err_word() {
    static int* ptrs[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!ptrs[dev]) {
        int* p = nullptr;
        if (error_word(&p) != cudaSuccess) return nullptr;
        ptrs[dev] = p;
    }
    return ptrs[dev];
}

static inline cudaStream_t as_stream(mq_stream s) { return reinterpret_cast<cudaStream_t>(s); }

static inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static mq_status launched(cudaError_t e, int kernels) {
    if (e != cudaSuccess) return MQ_ERR_CUDA;
    g_launches.fetch_add((uint64_t)kernels, std::memory_order_relaxed);
    return MQ_OK;
}

static bool nvfp4_shape_ok(int rows, int cols) { return rows > 0 && cols > 0 && cols % 64 == 0; }

extern "C" {

size_t mq_sf_swz_bytes(int rows, int cols) {
    if (rows <= 0 || cols <= 0 || cols % 64) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)(cols / 16);
}

size_t mq_weight_bytes(int N, int K) {
    if (N <= 0 || K <= 0 || N % 64 || K % 64) return 0;
    return (size_t)N * (size_t)(K / 2) + mq_sf_swz_bytes(N, K) + 16;
}

int mq_budget_blocks(int N, int K, double frac) {
    if (N <= 0 || K <= 0 || N % 64 || K % 64 || !(frac >= 0.0 && frac <= 1.0)) return -1;
    const double nb = (double)(N / 64) * (double)(K / 64);
    return (int)(frac * nb + 1e-9);
}

size_t mq_quantize_weight_workspace_bytes(int N, int K) {
    (void)N;
    (void)K;
    return (size_t)148 * 8 * sizeof(float);
}

size_t mq_delta_topk_workspace_bytes(int N, int K, int budget) {
    (void)N;
    (void)K;
    (void)budget;
    return 0;
}

size_t mq_gemm_workspace_bytes(int M, int N, int K, unsigned flags) {
    if (M <= 0 || N <= 0 || K <= 0 || N % 128 || K % 256) return 0;
    bool prefill = M > 128 && N % 256 == 0;
    if (flags & MQ_GEMM_DECODE) prefill = false;
    if (flags & MQ_GEMM_PREFILL) prefill = true;
    if (prefill) return 0;
    // mq_gemm's decode kernels (the small-problem one needs none, stream-K its partials)
    // and mq_gemm_act's (split-K): the larger of the two
    const size_t gemm_ws = plan_small(M, N, K) ? 0 : plan_streamk(M, N, K).ws;
    return std::max(gemm_ws, decode_workspace_bytes(M, N, K));
}

mq_status mq_quantize_weight(const mq_bf16* W, int N, int K, mq_nvfp4_mat* base, mq_nvfp4_mat* resid_full,
                             void* ws, size_t ws_bytes, mq_stream stream) {
    if (!W || !base || !resid_full || !nvfp4_shape_ok(N, K) || N % 64) return MQ_ERR_INVALID_ARG;
    if (!base->codes || !base->sf_swz || !base->gscale || !resid_full->codes || !resid_full->sf)
        return MQ_ERR_INVALID_ARG;
    if (base->rows != N || base->cols != K || resid_full->rows != N || resid_full->cols != K)
        return MQ_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(base->codes, 8) || !aligned(resid_full->codes, 8) || !aligned(base->sf_swz, 4))
        return MQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < mq_quantize_weight_workspace_bytes(N, K)) return MQ_ERR_WORKSPACE;
    cudaError_t e = launch_quant_weight(W, N, K, base->codes, base->sf, base->sf_swz, base->gscale,
                                        resid_full->codes, resid_full->sf, static_cast<float*>(ws),
                                        as_stream(stream));
    return launched(e, 2);
}

mq_status mq_hessian_diag(const mq_bf16* Xcal, int T, int K, float* H, mq_stream stream) {
    if (!Xcal || !H || T <= 0 || K <= 0 || K % 64 || !aligned(Xcal, 16)) return MQ_ERR_INVALID_ARG;
    if (T > hessian_max_tokens()) return MQ_ERR_UNSUPPORTED_SHAPE;
    return launched(launch_hessian(Xcal, T, K, H, as_stream(stream)), 1);
}

mq_status mq_delta_score_topk(const mq_bf16* W, const float* H, const mq_nvfp4_mat* base,
                              const mq_nvfp4_mat* resid_full, int budget, double* delta, int32_t* rank,
                              int32_t* sel, void* ws, size_t ws_bytes, mq_stream stream) {
    (void)resid_full;
    (void)ws;
    (void)ws_bytes;
    if (!W || !H || !base || !base->gscale || !delta) return MQ_ERR_INVALID_ARG;
    const int N = base->rows, K = base->cols;
    if (!nvfp4_shape_ok(N, K) || N % 64 || !aligned(W, 16)) return MQ_ERR_INVALID_ARG;
    const int B = (N / 64) * (K / 64);
    if (budget < 0 || budget > B) return MQ_ERR_INVALID_ARG;
    if (budget > 0 && (!rank || !sel)) return MQ_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    CUtensorMap tw;
    int* err = err_word();
    if (!err || !make_tmap_bf16_blocks(&tw, W, (uint64_t)K, (uint64_t)N)) return MQ_ERR_CUDA;
    cudaError_t e = launch_delta(tw, N, K, H, base->gscale, delta, err, s);
    if (e != cudaSuccess) return MQ_ERR_CUDA;
    g_launches.fetch_add(1);
    return launched(launch_topk(delta, B, budget, rank, sel, s), topk_launches(budget));
}

// X/xq (may be null): the whole-path call's activation rows, quantized by the same kernel
// after its strips (validated by the caller as mq_quantize_act does).
static mq_status quantize_weight_delta_impl(const mq_bf16* W, int N, int K, const float* H, mq_nvfp4_mat* base,
                                            mq_nvfp4_mat* resid_full, double* delta, void* ws, size_t ws_bytes,
                                            const mq_bf16* X, int M, mq_nvfp4_mat* xq, mq_stream stream) {
    if (!W || !H || !delta || !base || !nvfp4_shape_ok(N, K) || N % 64) return MQ_ERR_INVALID_ARG;
    if (!base->codes || !base->sf_swz || !base->gscale) return MQ_ERR_INVALID_ARG;
    if (base->rows != N || base->cols != K) return MQ_ERR_INVALID_ARG;
    if (resid_full && (!resid_full->codes || !resid_full->sf || resid_full->rows != N || resid_full->cols != K))
        return MQ_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(base->codes, 16) || !aligned(base->sf_swz, 16) ||
        (base->sf && !aligned(base->sf, 4)))
        return MQ_ERR_INVALID_ARG;
    if (resid_full && (!aligned(resid_full->codes, 16) || !aligned(resid_full->sf, 4))) return MQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < mq_quantize_weight_workspace_bytes(N, K)) return MQ_ERR_WORKSPACE;
    CUtensorMap tw;
    int* err = err_word();
    if (!err || !make_tmap_bf16_blocks(&tw, W, (uint64_t)K, (uint64_t)N)) return MQ_ERR_CUDA;
    cudaError_t e = launch_quant_delta(W, tw, N, K, H, base->codes, base->sf, base->sf_swz, base->gscale,
                                       resid_full ? resid_full->codes : nullptr, resid_full ? resid_full->sf : nullptr,
                                       delta, static_cast<float*>(ws), err, as_stream(stream), X, M,
                                       xq ? xq->codes : nullptr, xq ? xq->sf : nullptr, xq ? xq->sf_swz : nullptr,
                                       xq ? xq->gscale : nullptr);
    return launched(e, 2);
}

mq_status mq_quantize_weight_delta(const mq_bf16* W, int N, int K, const float* H, mq_nvfp4_mat* base,
                                   mq_nvfp4_mat* resid_full, double* delta, void* ws, size_t ws_bytes,
                                   mq_stream stream) {
    return quantize_weight_delta_impl(W, N, K, H, base, resid_full, delta, ws, ws_bytes, nullptr, 0, nullptr, stream);
}

mq_status mq_topk_blocks(const double* delta, int nblk, int budget, int32_t* rank, int32_t* sel, mq_stream stream) {
    if (!delta || nblk <= 0 || budget < 0 || budget > nblk) return MQ_ERR_INVALID_ARG;
    if (budget > 0 && (!rank || !sel)) return MQ_ERR_INVALID_ARG;
    return launched(launch_topk(delta, nblk, budget, rank, sel, as_stream(stream)), topk_launches(budget));
}

mq_status mq_pack_residual(const mq_nvfp4_mat* resid_full, const int32_t* sel, int budget, mq_residual_packed* out,
                           mq_stream stream) {
    if (!resid_full || !out || !resid_full->codes || !resid_full->sf) return MQ_ERR_INVALID_ARG;
    const int N = resid_full->rows, K = resid_full->cols;
    if (!nvfp4_shape_ok(N, K) || N % 64) return MQ_ERR_INVALID_ARG;
    if (out->N != N || out->K != K || out->nblk != budget || budget < 0 || budget > (N / 64) * (K / 64))
        return MQ_ERR_INVALID_ARG;
    if (!out->tile_ptr || !out->bitmap) return MQ_ERR_INVALID_ARG;
    if (budget > 0 && (!sel || !out->blk_codes || !out->blk_sf || !out->blk_kt)) return MQ_ERR_INVALID_ARG;
    if (budget > 0 && (!aligned(out->blk_codes, 16) || !aligned(out->blk_sf, 16))) return MQ_ERR_INVALID_ARG;
    return launched(launch_pack(resid_full->codes, resid_full->sf, N, K, sel, budget, out->blk_codes, out->blk_sf,
                                out->blk_kt, out->tile_ptr, out->bitmap, as_stream(stream)),
                    1);
}

static mq_status check_packed(const mq_residual_packed* out, int N, int K, const int32_t* sel, int budget) {
    if (!out || out->N != N || out->K != K || out->nblk != budget || budget < 0 || budget > (N / 64) * (K / 64))
        return MQ_ERR_INVALID_ARG;
    if (!out->tile_ptr || !out->bitmap) return MQ_ERR_INVALID_ARG;
    if (budget > 0 && (!sel || !out->blk_codes || !out->blk_sf || !out->blk_kt)) return MQ_ERR_INVALID_ARG;
    if (budget > 0 && (!aligned(out->blk_codes, 16) || !aligned(out->blk_sf, 16))) return MQ_ERR_INVALID_ARG;
    return MQ_OK;
}

// delta and rank: with rank != NULL the pack kernel also writes rank from sel and delta.
static mq_status pack_residual_weight_impl(const mq_bf16* W, const mq_nvfp4_mat* base, const int32_t* sel,
                                           int budget, mq_residual_packed* out, const double* delta,
                                           int32_t* rank, mq_stream stream) {
    if (!W || !base || !base->gscale) return MQ_ERR_INVALID_ARG;
    const int N = base->rows, K = base->cols;
    if (!nvfp4_shape_ok(N, K) || N % 64 || !aligned(W, 16)) return MQ_ERR_INVALID_ARG;
    const mq_status st = check_packed(out, N, K, sel, budget);
    if (st != MQ_OK) return st;
    return launched(launch_pack_w(W, N, K, base->gscale, sel, budget, out->blk_codes, out->blk_sf, out->blk_kt,
                                  out->tile_ptr, out->bitmap, delta, rank, as_stream(stream)),
                    1);
}

mq_status mq_pack_residual_weight(const mq_bf16* W, const mq_nvfp4_mat* base, const int32_t* sel, int budget,
                                  mq_residual_packed* out, mq_stream stream) {
    return pack_residual_weight_impl(W, base, sel, budget, out, nullptr, nullptr, stream);
}

mq_status mq_quantize_act(const mq_bf16* X, int M, int K, mq_nvfp4_mat* xq, mq_stream stream) {
    if (!X || !xq || !xq->codes || !xq->sf_swz || !xq->gscale || !nvfp4_shape_ok(M, K)) return MQ_ERR_INVALID_ARG;
    if (xq->rows != M || xq->cols != K || !aligned(X, 16) || !aligned(xq->codes, 8) || !aligned(xq->sf_swz, 4))
        return MQ_ERR_INVALID_ARG;
    if (K > 65536) return MQ_ERR_UNSUPPORTED_SHAPE;
    return launched(launch_quant_act(X, M, K, xq->codes, xq->sf, xq->sf_swz, xq->gscale, false, as_stream(stream)), 1);
}

// The whole-path call's activation quantizer: it quantizes X before waiting for the
// kernel preceding it (X is an input of that call, and the previous readers of xq are
// complete by the time any kernel of the call after the first one starts).
static mq_status quantize_act_early(const mq_bf16* X, int M, int K, mq_nvfp4_mat* xq, mq_stream stream) {
    if (!X || !xq || !xq->codes || !xq->sf_swz || !xq->gscale || !nvfp4_shape_ok(M, K)) return MQ_ERR_INVALID_ARG;
    if (xq->rows != M || xq->cols != K || !aligned(X, 16) || !aligned(xq->codes, 8) || !aligned(xq->sf_swz, 4))
        return MQ_ERR_INVALID_ARG;
    if (K > 65536) return MQ_ERR_UNSUPPORTED_SHAPE;
    return launched(launch_quant_act(X, M, K, xq->codes, xq->sf, xq->sf_swz, xq->gscale, true, as_stream(stream)), 1);
}

}  // extern "C"

namespace mq {

// The fused GEMM behind mq_gemm and mq_gemm_noalloc: argument checks, kernel choice (the
// flags, else prefill for M > 128 with N % 256 == 0), parameters, launch.
// prefetch: the caller guarantees wq and xq were complete before the GEMM could start (the
// whole-path call's order: the pack before it lets it start only after its own wait, and
// that wait already implies the activation quantizer and the quantize+Delta pass
// completed), so the decode kernel may load them before waiting for the pack.
// clear_counters: zero the workspace's tile counters on the stream before the kernel (a
// scratch that other calls share and that may hold anything).
mq_status gemm_dispatch(const mq_nvfp4_mat* xq, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y,
                        int M, int N, int K, unsigned flags, void* ws, size_t ws_bytes, bool prefetch,
                        bool clear_counters, mq_stream stream) {
    if (!xq || !wq || !Y || M <= 0 || N <= 0 || K <= 0 || N % 64 || K % 64) return MQ_ERR_INVALID_ARG;
    if (N % 128 || K % 256) return MQ_ERR_UNSUPPORTED_SHAPE;
    if (!xq->codes || !xq->sf_swz || !xq->gscale || !wq->codes || !wq->sf_swz || !wq->gscale)
        return MQ_ERR_INVALID_ARG;
    if (xq->rows != M || xq->cols != K || wq->rows != N || wq->cols != K) return MQ_ERR_INVALID_ARG;
    if ((flags & MQ_GEMM_BASE_ONLY) && (flags & MQ_GEMM_RESIDUAL_ONLY)) return MQ_ERR_INVALID_ARG;
    if (!aligned(xq->codes, 16) || !aligned(wq->codes, 16) || !aligned(xq->sf_swz, 16) || !aligned(wq->sf_swz, 16))
        return MQ_ERR_INVALID_ARG;
    const bool has_r = r && r->nblk > 0 && !(flags & MQ_GEMM_BASE_ONLY);
    if (r && r->nblk > 0) {
        if (r->N != N || r->K != K || !r->blk_codes || !r->blk_sf || !r->tile_ptr || !r->bitmap)
            return MQ_ERR_INVALID_ARG;
        if (!aligned(r->blk_codes, 16) || !aligned(r->blk_sf, 16)) return MQ_ERR_INVALID_ARG;
    }
    // kernel choice: the prefill kernel tiles 256 weight rows, the decode kernel 128
    bool prefill = M > 128 && N % 256 == 0;
    if (flags & MQ_GEMM_DECODE) prefill = false;
    if (flags & MQ_GEMM_PREFILL) {
        if (N % 256) return MQ_ERR_UNSUPPORTED_SHAPE;
        prefill = true;
    }
    GemmParams p;
    memset(&p, 0, sizeof p);
    p.w_sf = wq->sf_swz;
    p.x_sf = xq->sf_swz;
    p.g_w = wq->gscale;
    p.g_x = xq->gscale;
    if (has_r) {
        p.blk_codes = r->blk_codes;
        p.blk_sf = r->blk_sf;
        p.tile_ptr = r->tile_ptr;
        p.bitmap = r->bitmap;
    }
    p.has_resid = has_r ? 1 : 0;
    p.nblk = has_r ? r->nblk : 0;
    p.Y = Y;
    p.M = M;
    p.N = N;
    p.K = K;
    p.mode = (flags & MQ_GEMM_BASE_ONLY) ? 1 : (flags & MQ_GEMM_RESIDUAL_ONLY) ? 2 : 0;
    p.prefetch = prefetch ? 1 : 0;
    p.w_ready = (flags & MQ_GEMM_WEIGHTS_READY) ? 1 : 0;
    CUtensorMap tw, tx;
    if (prefill) {
        // CTA pairs: each CTA stages 128 tokens and 128 of the tile's 256 weight rows
        CUtensorMap twsf, txsf, trc, trsf;
        const uint64_t KS64 = (uint64_t)K / 64;
        if (!make_tmap_bytes(&tw, wq->codes, (uint64_t)K / 2, (uint64_t)N, 128, 128)) return MQ_ERR_CUDA;
        if (!make_tmap_bytes(&tx, xq->codes, (uint64_t)K / 2, (uint64_t)M, 128, 128)) return MQ_ERR_CUDA;
        if (!make_tmap_u32(&twsf, wq->sf_swz, 128, (uint64_t)((N + 127) / 128) * KS64, 128, 4)) return MQ_ERR_CUDA;
        if (!make_tmap_u32(&txsf, xq->sf_swz, 128, (uint64_t)((M + 127) / 128) * KS64, 128, 4)) return MQ_ERR_CUDA;
        // without a residual these two maps are never used: any valid buffer will do
        const void* rc = has_r ? (const void*)r->blk_codes : (const void*)xq->sf_swz;
        const void* rs = has_r ? (const void*)r->blk_sf : (const void*)xq->sf_swz;
        const uint64_t nb = has_r ? (uint64_t)r->nblk : 1;
        if (!make_tmap_u32(&trc, rc, 256, has_r ? 2 * nb : 1, 256, 1)) return MQ_ERR_CUDA;
        if (!make_tmap_u32(&trsf, rs, 128, nb, 128, 1)) return MQ_ERR_CUDA;
        return launched(launch_gemm_prefill2(tw, tx, twsf, txsf, trc, trsf, p, as_stream(stream)), 1);
    }
    p.wait_ns = 2000000000ull;
    p.skip_unit = -1;
    const int fault_unit = g_fault_unit.exchange(-1);
    if (fault_unit >= 0) {
        p.skip_unit = fault_unit;
        p.wait_ns = g_fault_ns.load();
    }
    if (const int S = plan_small(M, N, K)) {
        // small problems: each tile split among the CTAs of one cluster, no workspace
        if (!make_tmap_bytes(&tw, wq->codes, (uint64_t)K / 2, (uint64_t)N, 128, 128)) return MQ_ERR_CUDA;
        if (!make_tmap_bytes(&tx, xq->codes, (uint64_t)K / 2, (uint64_t)M, 128, M <= 16 ? 16 : 32))
            return MQ_ERR_CUDA;
        return launched(launch_gemm_small(tw, tx, p, S, as_stream(stream)), 1);
    }
    const StreamKPlan d = plan_streamk(M, N, K);
    // the kernel splits the units with 32-bit arithmetic (units x grid < 2^32)
    if ((int64_t)d.units * d.grid >= (int64_t(1) << 32)) return MQ_ERR_UNSUPPORTED_SHAPE;
    const size_t need = d.ws;
    if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return MQ_ERR_WORKSPACE;
    if (!make_tmap_bytes(&tw, wq->codes, (uint64_t)K / 2, (uint64_t)N, 128, 128)) return MQ_ERR_CUDA;
    if (!make_tmap_bytes(&tx, xq->codes, (uint64_t)K / 2, (uint64_t)M, 128, (uint32_t)d.BN)) return MQ_ERR_CUDA;
    if (need > 0) {
        p.partial = static_cast<float*>(ws);
        p.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + d.slots_bytes);
        if (clear_counters &&
            cudaMemsetAsync(p.counters, 0, (size_t)d.tiles_m * d.tiles_n * sizeof(int), as_stream(stream)) !=
                cudaSuccess)
            return MQ_ERR_CUDA;
    }
    return launched(launch_gemm_streamk(tw, tx, p, d, as_stream(stream)), 1);
}

}  // namespace mq

extern "C" {

mq_status mq_gemm(const mq_nvfp4_mat* xq, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y, int M,
                  int N, int K, unsigned flags, void* ws, size_t ws_bytes, mq_stream stream) {
    return gemm_dispatch(xq, wq, r, Y, M, N, K, flags, ws, ws_bytes, false, false, stream);
}

// Decode kernel with the activation quantization inside it (X bf16).
static mq_status gemm_act_impl(const mq_bf16* X, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y,
                               int M, int N, int K, unsigned flags, void* ws, size_t ws_bytes, float* gx_out,
                               bool prefetch, mq_stream stream) {
    if (!X || !wq || !Y || M <= 0 || N <= 0 || K <= 0 || N % 64 || K % 64) return MQ_ERR_INVALID_ARG;
    if (N % 128 || K % 256 || (flags & MQ_GEMM_PREFILL)) return MQ_ERR_UNSUPPORTED_SHAPE;
    if (!wq->codes || !wq->sf_swz || !wq->gscale || wq->rows != N || wq->cols != K) return MQ_ERR_INVALID_ARG;
    if ((flags & MQ_GEMM_BASE_ONLY) && (flags & MQ_GEMM_RESIDUAL_ONLY)) return MQ_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(wq->codes, 16) || !aligned(wq->sf_swz, 16)) return MQ_ERR_INVALID_ARG;
    const bool has_r = r && r->nblk > 0 && !(flags & MQ_GEMM_BASE_ONLY);
    if (r && r->nblk > 0) {
        if (r->N != N || r->K != K || !r->blk_codes || !r->blk_sf || !r->tile_ptr || !r->bitmap)
            return MQ_ERR_INVALID_ARG;
        if (!aligned(r->blk_codes, 16) || !aligned(r->blk_sf, 16)) return MQ_ERR_INVALID_ARG;
    }
    GemmParams p;
    memset(&p, 0, sizeof p);
    p.w_sf = wq->sf_swz;
    p.g_w = wq->gscale;
    if (has_r) {
        p.blk_codes = r->blk_codes;
        p.blk_sf = r->blk_sf;
        p.tile_ptr = r->tile_ptr;
        p.bitmap = r->bitmap;
    }
    p.has_resid = has_r ? 1 : 0;
    p.nblk = has_r ? r->nblk : 0;
    p.Y = Y;
    p.M = M;
    p.N = N;
    p.K = K;
    p.mode = (flags & MQ_GEMM_BASE_ONLY) ? 1 : (flags & MQ_GEMM_RESIDUAL_ONLY) ? 2 : 0;
    p.prefetch = prefetch ? 1 : 0;
    p.x_bf16 = X;
    p.gx_out = gx_out;
    DecodePlan d = plan_decode(M, N, K);
    const size_t need = decode_workspace_bytes(M, N, K);
    if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return MQ_ERR_WORKSPACE;
    CUtensorMap tw;
    if (!make_tmap_bytes(&tw, wq->codes, (uint64_t)K / 2, (uint64_t)N, 128, 128)) return MQ_ERR_CUDA;
    if (need > 0) {
        size_t part = (size_t)d.splits * d.tiles_m * d.BN * N * sizeof(float);
        part = (part + 255) & ~size_t(255);
        p.partial = static_cast<float*>(ws);
        p.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + part);
    }
    // the X tensor map is not used in this mode
    return launched(launch_gemm_decode(tw, tw, p, d, as_stream(stream)), 1);
}

mq_status mq_gemm_act(const mq_bf16* X, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y, int M, int N,
                      int K, unsigned flags, void* ws, size_t ws_bytes, float* gx_out, mq_stream stream) {
    return gemm_act_impl(X, wq, r, Y, M, N, K, flags, ws, ws_bytes, gx_out, false, stream);
}

mq_status mq_run_layer(const mq_bf16* W, const mq_bf16* X, const mq_bf16* Xcal, mq_bf16* Y, int M, int N, int K,
                       int T, int budget, unsigned flags, int host, mq_layer_buffers* buf, mq_stream stream) {
    const bool prepared = (flags & MQ_LAYER_PREPARED) != 0;
    flags &= ~(unsigned)MQ_LAYER_PREPARED;
    if (prepared) {
        // inference on a prepared layer: A6 + A7 + A8 (X in, Y out)
        if (!X || !Y || !buf || M <= 0 || N <= 0 || K <= 0) return MQ_ERR_INVALID_ARG;
        if (buf->packed.nblk != budget) return MQ_ERR_INVALID_ARG;
        cudaStream_t s = as_stream(stream);
        const mq_bf16* x = X;
        mq_bf16* y = Y;
        if (host) {
            if (!buf->X_dev || !buf->Y_dev) return MQ_ERR_INVALID_ARG;
            if (cudaMemcpyAsync(buf->X_dev, X, (size_t)M * K * 2, cudaMemcpyHostToDevice, s) != cudaSuccess)
                return MQ_ERR_CUDA;
            x = buf->X_dev;
            y = buf->Y_dev;
        }
        mq_status st;
        if ((st = mq_quantize_act(x, M, K, &buf->xq, stream)) != MQ_OK) return st;
        if ((st = gemm_dispatch(&buf->xq, &buf->base, &buf->packed, y, M, N, K, flags, buf->ws_gemm,
                                buf->ws_gemm_bytes, false, false, stream)) != MQ_OK)
            return st;
        if (host && cudaMemcpyAsync(Y, buf->Y_dev, (size_t)M * N * 2, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return MQ_ERR_CUDA;
        return MQ_OK;
    }
    if (!W || !X || !Xcal || !Y || !buf || M <= 0 || N <= 0 || K <= 0 || T <= 0) return MQ_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const mq_bf16 *w = W, *x = X, *xc = Xcal;
    mq_bf16* y = Y;
    if (host) {
        if (!buf->W_dev || !buf->X_dev || !buf->Xcal_dev || !buf->Y_dev) return MQ_ERR_INVALID_ARG;
        if (cudaMemcpyAsync(buf->W_dev, W, (size_t)N * K * 2, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(buf->Xcal_dev, Xcal, (size_t)T * K * 2, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(buf->X_dev, X, (size_t)M * K * 2, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return MQ_ERR_CUDA;
        w = buf->W_dev;
        x = buf->X_dev;
        xc = buf->Xcal_dev;
        y = buf->Y_dev;
    }
    // The method's order, with the activation quantizer moved ahead of top-K. Every kernel
    // waits for its predecessor before reading its outputs. The weight maxima pass and the
    // activation quantizer read only inputs of this call: they let their dependent start
    // at once, do their work and wait at their end (so their completion still implies
    // their predecessor's). The others let their dependent start right after their wait.
    // When the GEMM starts, the quantize+Delta kernel and the activation quantizer have
    // completed, and the GEMM requests W and X before waiting for its predecessor
    // (prefetch). The activation quantizer runs as its
    // own kernel: on B200 at decode sizes that is faster than quantizing inside the GEMM
    // (mq_gemm_act), whose per-token maxima must first be exchanged between the K splits.
    mq_status st;
    if ((st = mq_hessian_diag(xc, T, K, buf->H, stream)) != MQ_OK) return st;
    // A6 rides on the quantize+Delta kernel when its CTAs can hold a row (K <= 4096): its
    // CTAs with the fewest strips quantize the activation rows at the end; otherwise the
    // activation quantizer runs as its own kernel in early mode
    mq_nvfp4_mat* xq = &buf->xq;
    if (!x || !xq->codes || !xq->sf_swz || !xq->gscale || xq->rows != M || xq->cols != K || !aligned(x, 16) ||
        !aligned(xq->codes, 8) || !aligned(xq->sf_swz, 4))
        return MQ_ERR_INVALID_ARG;
    const bool act_in_qd = quant_delta_takes_act(K);
    if ((st = quantize_weight_delta_impl(w, N, K, buf->H, &buf->base, nullptr, buf->delta, buf->ws_quant,
                                         buf->ws_quant_bytes, act_in_qd ? x : nullptr, M, act_in_qd ? xq : nullptr,
                                         stream)) != MQ_OK)
        return st;
    if (!act_in_qd && (st = quantize_act_early(x, M, K, xq, stream)) != MQ_OK) return st;
    // A4 as two parts: the selection kernel writes sel, and rank (which the GEMM does not
    // read) is written by extra CTAs of the pack kernel, beside the packing
    {
        const int nblk = (N / 64) * (K / 64);
        if (!buf->delta || budget < 0 || budget > nblk || (budget > 0 && (!buf->rank || !buf->sel)))
            return MQ_ERR_INVALID_ARG;
        if ((st = launched(launch_topk_select(buf->delta, nblk, budget, buf->sel, s), budget > 0 ? 1 : 0)) != MQ_OK)
            return st;
    }
    if ((st = pack_residual_weight_impl(w, &buf->base, buf->sel, budget, &buf->packed, buf->delta, buf->rank,
                                        stream)) != MQ_OK)
        return st;
    if ((st = gemm_dispatch(&buf->xq, &buf->base, &buf->packed, y, M, N, K, flags, buf->ws_gemm, buf->ws_gemm_bytes,
                            true, false, stream)) != MQ_OK)
        return st;
    if (host && cudaMemcpyAsync(Y, buf->Y_dev, (size_t)M * N * 2, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MQ_ERR_CUDA;
    return MQ_OK;
}

mq_status mq_smooth_scales(const mq_bf16* Xcal, int T, const mq_bf16* W, int N, int K, float* s, mq_stream stream) {
    if (!Xcal || !W || !s || T <= 0 || N <= 0 || K <= 0 || K % 64) return MQ_ERR_INVALID_ARG;
    if (!aligned(Xcal, 16) || !aligned(W, 16)) return MQ_ERR_INVALID_ARG;
    return launched(launch_smooth_scales(Xcal, T, W, N, K, s, as_stream(stream)), 1);
}

mq_status mq_smooth_apply(const mq_bf16* A, int rows, int K, const float* s, int invert, mq_bf16* out,
                          mq_stream stream) {
    if (!A || !s || !out || rows <= 0 || K <= 0 || K % 64) return MQ_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(out, 16)) return MQ_ERR_INVALID_ARG;
    return launched(launch_smooth_apply(A, rows, K, s, invert ? 1 : 0, out, as_stream(stream)), 1);
}

mq_status mq_get_error(mq_stream stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MQ_ERR_CUDA;
    int v = 0;
    if (read_clear_error(&v) != cudaSuccess) return MQ_ERR_CUDA;
    return v ? (mq_status)v : MQ_OK;
}

const char* mq_status_string(mq_status s) {
    switch (s) {
        case MQ_OK: return "ok";
        case MQ_ERR_INVALID_ARG: return "invalid argument";
        case MQ_ERR_UNSUPPORTED_SHAPE: return "shape not supported by the GEMM kernels";
        case MQ_ERR_WORKSPACE: return "workspace missing or too small";
        case MQ_ERR_CUDA: return "CUDA error";
        case MQ_ERR_TIMEOUT: return "device pipeline wait timed out";
    }
    return "unknown status";
}

uint64_t mq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

mq_status mq_test_arm_wait_fault(int unit, double wait_ms) {
    if (unit < 0 || !(wait_ms >= 0.01 && wait_ms <= 2000.0)) return MQ_ERR_INVALID_ARG;
    g_fault_ns.store((unsigned long long)(wait_ms * 1e6));
    g_fault_unit.store(unit);
    return MQ_OK;
}

}  // extern "C"

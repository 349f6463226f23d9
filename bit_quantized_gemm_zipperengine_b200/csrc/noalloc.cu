// mq_gemm_noalloc: the fused GEMM for callers that cannot allocate device memory.
//
// Some callers of this library have no way to obtain a device workspace: code embedded
// in a host framework whose device memory is owned by that framework's allocator and
// that exposes no workspace hook, or latency-critical paths where an allocation (and
// the synchronization it may imply) is not allowed. For them this entry point takes
// only inputs and outputs; the decode kernel's split-K scratch (fp32 partials and
// per-tile counters) lives in one file-scope device array of this library instead.
//
// The array is kNoallocScratchBytes (8 MiB) on every GPU that loads the library, held
// until the process exits. All calls share it: calls that overlap on the GPU (other
// streams, other threads) race on it and must be serialized by the caller.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(8) << 20;

// The scratch. In host code this name is only a stand-in for the device symbol: its
// device address comes from cudaGetSymbolAddress (per device) below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_dev[64] = {};  // device address of the scratch, per device ordinal

// Set-up, once per device, with that device current: look up the array's address.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_dev[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_dev[dev] = p;
    }
    *out = g_scratch_dev[dev];
    return cudaSuccess;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool tmap_bytes(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_bytes,
                uint32_t box_rows) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_bytes, box_rows};
    cuuint32_t es[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool al(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" {

size_t mq_gemm_noalloc_scratch_limit(void) { return kNoallocScratchBytes; }

mq_status mq_gemm_noalloc(const mq_nvfp4_mat* xq, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y,
                          int M, int N, int K, unsigned flags, mq_stream stream) {
    using namespace mq;
    if (!xq || !wq || !Y || M <= 0 || N <= 0 || K <= 0 || N % 64 || K % 64) return MQ_ERR_INVALID_ARG;
    if (N % 128 || K % 256) return MQ_ERR_UNSUPPORTED_SHAPE;
    if (!xq->codes || !xq->sf_swz || !xq->gscale || !wq->codes || !wq->sf_swz || !wq->gscale)
        return MQ_ERR_INVALID_ARG;
    if (xq->rows != M || xq->cols != K || wq->rows != N || wq->cols != K) return MQ_ERR_INVALID_ARG;
    if ((flags & MQ_GEMM_BASE_ONLY) && (flags & MQ_GEMM_RESIDUAL_ONLY)) return MQ_ERR_INVALID_ARG;
    if (!al(xq->codes, 16) || !al(wq->codes, 16) || !al(xq->sf_swz, 16) || !al(wq->sf_swz, 16))
        return MQ_ERR_INVALID_ARG;
    const bool has_r = r && r->nblk > 0 && !(flags & MQ_GEMM_BASE_ONLY);
    if (r && r->nblk > 0) {
        if (r->N != N || r->K != K || !r->blk_codes || !r->blk_sf || !r->tile_ptr || !r->bitmap)
            return MQ_ERR_INVALID_ARG;
        if (!al(r->blk_codes, 16) || !al(r->blk_sf, 16)) return MQ_ERR_INVALID_ARG;
    }
    const DecodePlan d = plan_decode(M, N, K);
    const size_t need = decode_workspace_bytes(M, N, K);
    if (need > kNoallocScratchBytes) return MQ_ERR_WORKSPACE;  // beyond the static scratch

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    GemmParams p;
    memset(&p, 0, sizeof p);
    if (need > 0) {
        void* scratch = nullptr;
        if (scratch_address(&scratch) != cudaSuccess) return MQ_ERR_CUDA;
        size_t part = (size_t)d.splits * d.tiles_m * d.BN * N * sizeof(float);
        part = (part + 255) & ~size_t(255);
        p.partial = static_cast<float*>(scratch);
        p.counters = reinterpret_cast<int*>(static_cast<unsigned char*>(scratch) + part);
        // the tile counters must start at zero; the array keeps the last call's contents
        if (cudaMemsetAsync(p.counters, 0, (size_t)d.tiles_m * d.tiles_n * sizeof(int), s) != cudaSuccess)
            return MQ_ERR_CUDA;
    }
    CUtensorMap tw, tx;
    if (!tmap_bytes(&tw, wq->codes, (uint64_t)K / 2, (uint64_t)N, 128, 128)) return MQ_ERR_CUDA;
    if (!tmap_bytes(&tx, xq->codes, (uint64_t)K / 2, (uint64_t)M, 128, (uint32_t)d.BN)) return MQ_ERR_CUDA;
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
    p.Y = Y;
    p.M = M;
    p.N = N;
    p.K = K;
    p.mode = (flags & MQ_GEMM_BASE_ONLY) ? 1 : (flags & MQ_GEMM_RESIDUAL_ONLY) ? 2 : 0;
    return launch_gemm_decode(tw, tx, p, d, s) == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}

}  // extern "C"

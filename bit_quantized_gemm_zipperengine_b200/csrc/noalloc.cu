// mq_gemm_noalloc: the fused GEMM for callers that cannot allocate device memory.
//
// Some callers of this library have no way to obtain a device workspace: code embedded
// in a host framework whose device memory is owned by that framework's allocator and
// that exposes no workspace hook, or latency-critical paths where an allocation (and
// the synchronization it may imply) is not allowed. For them this entry point takes
// only inputs and outputs; the decode kernel's split-K scratch (fp32 partials and
// per-tile counters) lives in one file-scope device array of this library instead.
//
// The array is kNoallocScratchBytes (16 MiB) on every GPU that loads the library, held
// until the process exits. All calls share it: calls that overlap on the GPU (other
// streams, other threads) race on it and must be serialized by the caller.
#include <mutex>

#include "common.cuh"
#include "gemm.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(16) << 20;

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

}  // namespace

extern "C" {

size_t mq_gemm_noalloc_scratch_limit(void) { return kNoallocScratchBytes; }

mq_status mq_gemm_noalloc(const mq_nvfp4_mat* xq, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y,
                          int M, int N, int K, unsigned flags, mq_stream stream) {
    // the same kernel choice as mq_gemm (flags, else by shape); only the decode kernel's
    // split-K reduction needs scratch, and a problem needing more than the static array
    // holds is refused before anything is launched
    const size_t need = mq_gemm_workspace_bytes(M, N, K, flags);
    if (need > kNoallocScratchBytes) return MQ_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0 && scratch_address(&scratch) != cudaSuccess) return MQ_ERR_CUDA;
    // the array keeps the last call's contents: the tile counters are cleared on the stream
    return mq::gemm_dispatch(xq, wq, r, Y, M, N, K, flags, scratch, need > 0 ? kNoallocScratchBytes : 0, false, true,
                             stream);
}

}  // extern "C"

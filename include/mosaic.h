/*
 * mosaic.h -- C ABI of libmosaic, the B200 (sm_100a) MosaicQuant / ZipperEngine path.
 *
 * The method (MosaicQuant technical summary, "Methodology"; arXiv 2606.15652 abstract):
 * the weight matrix W is split into a dense 4-bit base Q(W) plus a 4-bit residual R,
 * W ~ Q(W) + R (section 1, "Inlier-outlier disaggregation"); R is kept only on the
 * top-K 64x64 blocks ranked by a Hessian-guided Delta-score (section 2, "Block-wise
 * residual allocation"); ZipperEngine runs base and sparse residual in one fused GEMM,
 * with activation quantization and the reduce-sum in the same pipeline (section 3).
 *
 * Number format (NVFP4): E2M1 values {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit, one
 * E4M3 scale per 16 consecutive K elements, and an fp32 tensor scale g (one per weight
 * matrix, one per token for activations). g = amax / 2688 (1 if amax = 0). Per group:
 * s = amax_group / (6 g); sf = E4M3_rne_satfinite(s); d = dec(sf) * g; r = 1 / d;
 * code_i = E2M1_rne_satfinite(a_i * r) (a signed zero when d = 0). Each step is one fp32
 * IEEE operation with round-to-nearest-even, none contracted into a fused multiply-add;
 * codes and scales are bit-exact with the CPU oracle. The Delta-score is computed in
 * fp64 (see mq_delta_score_topk).
 *
 * Conventions for every call:
 *  - All pointers are DEVICE pointers unless stated otherwise; the caller allocates and
 *    frees every buffer. The library allocates no device memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *    The returned status covers argument validation and launch errors only; a device
 *    side timeout (a pipeline wait that gave up) is reported by mq_get_error().
 *  - Shapes: N and K must be multiples of 64 (MQ_ERR_INVALID_ARG otherwise); the GEMM
 *    additionally needs N % 128 == 0 and K % 256 == 0 (MQ_ERR_UNSUPPORTED_SHAPE).
 *    M >= 1. Inputs must be finite (NaN/Inf is a precondition violation).
 *  - bf16 buffers are passed as raw 16-bit patterns (mq_bf16).
 */
#ifndef MOSAIC_H_
#define MOSAIC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t mq_bf16;
typedef void* mq_stream; /* cudaStream_t */

typedef enum {
    MQ_OK = 0,
    MQ_ERR_INVALID_ARG = 1,       /* null pointer, bad shape, budget out of range */
    MQ_ERR_UNSUPPORTED_SHAPE = 2, /* valid NVFP4 shape the GEMM kernels do not tile */
    MQ_ERR_WORKSPACE = 3,         /* workspace missing or smaller than required */
    MQ_ERR_CUDA = 4,              /* a CUDA runtime/driver call or launch failed */
    MQ_ERR_TIMEOUT = 5            /* a device pipeline wait gave up (see mq_get_error) */
} mq_status;

/* GEMM flags. */
enum {
    MQ_GEMM_AUTO = 0,          /* prefill kernel for M > 128 and N % 256 == 0, else decode */
    MQ_GEMM_DECODE = 1,        /* small-M kernel: W as the MMA's M side, split-K */
    MQ_GEMM_PREFILL = 2,       /* large-M kernel: X as the MMA's M side; needs N % 256 == 0 */
    MQ_GEMM_BASE_ONLY = 4,     /* skip the residual blocks (dense-only reference) */
    MQ_GEMM_RESIDUAL_ONLY = 8, /* only the residual blocks (linearity check) */
    MQ_LAYER_PREPARED = 16,    /* mq_run_layer only: the weight is already prepared (see there) */
    MQ_GEMM_WEIGHTS_READY = 32 /* the weight is complete before this call (see mq_gemm) */
};

/*
 * An NVFP4 matrix, rows x cols (weights: N x K; activations: M x K).
 *  codes : [rows][cols/2] bytes; element 2j of a row in the low nibble of byte j,
 *          element 2j+1 in the high nibble. Nibble = sign (bit 3) | E2M1 magnitude.
 *  sf    : [rows][cols/16] E4M3 bytes, row-major (group q of row r at r*cols/16 + q).
 *          May be NULL where a call says so.
 *  sf_swz: the GEMM's tiled scale layout, mq_sf_swz_bytes(rows, cols) bytes: rows in
 *          tiles of 128 and groups in steps of 4 (64 K elements); each (row tile,
 *          K step) is a 512-byte chunk at ((r/128)*(cols/64) + q/4)*512, and inside it
 *          row t = r%128, group q%4 sit at (t%32)*16 + (t/32)*4 + q%4. Rows past `rows`
 *          up to the next multiple of 128 hold zero.
 *  gscale: fp32 tensor scale(s): [1] for weights, [rows] for activations.
 */
typedef struct {
    int rows;
    int cols;
    uint8_t* codes;
    uint8_t* sf;
    uint8_t* sf_swz;
    float* gscale;
} mq_nvfp4_mat;

/*
 * Packed sparse residual of an N x K weight, nblk selected blocks in ascending block
 * index b = nt*(K/64) + kt (nt = block row, kt = block column).
 *  blk_codes: [nblk][2048]; block row r (0..63), packed byte j (0..31) of that row at
 *             (r/8)*256 + (j/16)*128 + (r%8)*16 + (j%16) (8-row x 16-byte core
 *             matrices, the MMA's no-swizzle K-major operand layout).
 *  blk_sf   : [nblk][512]; the block's 64x4 scales written into the 128-row scale chunk
 *             of its 128-row band (tile row t = 64*(nt%2) + r, group q at
 *             (t%32)*16 + (t/32)*4 + q), every other byte zero.
 *  blk_kt   : [nblk] block column of each entry.
 *  tile_ptr : [N/64 + 1] CSR over block rows: entries of block row nt are
 *             [tile_ptr[nt], tile_ptr[nt+1]).
 *  bitmap   : [N/64][ceil((K/64)/32)] u32; bit kt%32 of word kt/32 set iff (nt, kt)
 *             is selected.
 */
typedef struct {
    int N;
    int K;
    int nblk;
    uint8_t* blk_codes;
    uint8_t* blk_sf;
    int32_t* blk_kt;
    int32_t* tile_ptr;
    uint32_t* bitmap;
} mq_residual_packed;

/* ---- sizes (host only, no device work) ---------------------------------------- */

/* Bytes of an sf_swz buffer for a rows x cols matrix: ceil(rows/128)*128*(cols/16). */
size_t mq_sf_swz_bytes(int rows, int cols);

/*
 * Bytes of one GEMM-ready NVFP4 weight (the base Q(W) that mq_gemm reads), for a caller
 * that allocates it as one buffer: codes (N*K/2 bytes) at offset 0, sf_swz
 * (mq_sf_swz_bytes(N, K) bytes) at offset N*K/2, and the fp32 tensor scale at offset
 * N*K/2 + mq_sf_swz_bytes(N, K), padded to 16 bytes. Every offset is a multiple of 16
 * for a 16-byte aligned buffer, as the calls require. The optional linear scales
 * (sf, N*K/16 bytes), the full residual of mq_quantize_weight and the packed residual
 * are separate buffers. 0 on a bad shape (N, K <= 0 or not multiples of 64).
 */
size_t mq_weight_bytes(int N, int K);

/* floor(frac * (N/64) * (K/64)); -1 on a bad shape or frac outside [0, 1]. */
int mq_budget_blocks(int N, int K, double frac);

/* Workspace of mq_quantize_weight (per-CTA partial maxima). */
size_t mq_quantize_weight_workspace_bytes(int N, int K);

/* Workspace of mq_delta_score_topk for `budget` selected blocks. */
size_t mq_delta_topk_workspace_bytes(int N, int K, int budget);

/* Workspace of mq_gemm and mq_gemm_act: fp32 partials of the output tiles whose K range
 * is split between CTAs, plus per-tile counters (0 when the large-M kernel runs or no
 * tile is split). The size depends on the current device's SM count. The counter region
 * must be zero before the first call on a workspace; every call leaves it zero again
 * when it completes (a call that ended in MQ_ERR_TIMEOUT may not: zero it again). Calls
 * sharing a workspace must not overlap on the GPU. */
size_t mq_gemm_workspace_bytes(int M, int N, int K, unsigned flags);

/* ---- the path ----------------------------------------------------------------- */

/*
 * A0. Equivalent transform ahead of quantization (MosaicQuant summary, "Methodology",
 * section 1: activation outliers are migrated into the weights by an equivalent
 * transform such as SmoothQuant; the pages name it without defining it). SmoothQuant's
 * per-input-channel rule with migration strength 1/2:
 *   s_k = fp32( sqrt( fp32( max_t |Xcal[t][k]| / max_n |W[n][k]| ) ) )  (1 if either is 0),
 * each operation IEEE with round-to-nearest-even. Xcal: bf16 [T][K], W: bf16 [N][K], both
 * 16-byte aligned; s: fp32 [K]. K % 64 == 0.
 */
mq_status mq_smooth_scales(const mq_bf16* Xcal, int T, const mq_bf16* W, int N, int K, float* s, mq_stream stream);

/*
 * Applies the transform: out = bf16_rn(A[r][k] * s_k) for a weight (invert = 0) or
 * bf16_rn(A[r][k] / s_k) for activations (invert != 0), so that X W^T = X' W'^T up to the
 * two bf16 roundings. A, out: bf16 [rows][K], 16-byte aligned (out may equal A).
 */
mq_status mq_smooth_apply(const mq_bf16* A, int rows, int K, const float* s, int invert, mq_bf16* out,
                          mq_stream stream);

/*
 * A1. Weight quantization (MosaicQuant summary, "Methodology", section 1).
 * W: bf16 [N][K]. Writes base = NVFP4(W, g_w) and resid_full = NVFP4(W - deq Q(W), g_w)
 * for EVERY element (the residual uses the base's tensor scale g_w; selection happens
 * later). base: codes, sf_swz and gscale[1] required, sf optional (NULL skips it).
 * resid_full: codes and sf required; its sf_swz is not written; its gscale may be NULL
 * (the residual shares base->gscale). ws: mq_quantize_weight_workspace_bytes.
 */
mq_status mq_quantize_weight(const mq_bf16* W, int N, int K, mq_nvfp4_mat* base, mq_nvfp4_mat* resid_full,
                             void* ws, size_t ws_bytes, mq_stream stream);

/*
 * A2. Diagonal Hessian estimate of the input channels (summary, "Methodology",
 * section 2): H_k = fp32( S_k / T ), S_k the fp64 sum of the squares fp64(x_tk)^2 by a
 * fixed pairwise tree over t (the T squares padded with zeros to the next power of two
 * P, then v[i] += v[i+h] for h = P/2, ..., 1). Xcal: bf16 [T][K], H: fp32 [K].
 * 1 <= T <= 1024 calibration tokens (MQ_ERR_UNSUPPORTED_SHAPE above), K % 64 == 0,
 * Xcal 16-byte aligned (MQ_ERR_INVALID_ARG otherwise).
 */
mq_status mq_hessian_diag(const mq_bf16* Xcal, int T, int K, float* H, mq_stream stream);

/*
 * A3 + A4. Delta-score and top-K block selection (summary, "Methodology", section 2:
 * marginal reduction of the output distortion per block, residual error weighted by
 * the diagonal Hessian). For block b = (nt, kt):
 *   Delta_b = T64_k( fp64(H_k) * T64_r( fp64(e)*fp64(e) - fp64(e')*fp64(e') ) ),
 *   e = fp32(W - deq Q(W)), e' = fp32(e - deq R),
 * where T64 is the pairwise tree v[i] += v[i+32], +16, +8, +4, +2, +1 over the block's
 * 64 rows (inner) and 64 columns (outer), every add and multiply in fp64 with
 * round-to-nearest-even. Both squares are exact in fp64, so each element's term is
 * rounded once (the kernel takes it as one fp64 fused multiply-add, e*e - (e'*e'),
 * which gives the same bits). The kernel recomputes e and e' from W and the
 * tensor scale base->gscale, bit-identical to mq_quantize_weight's codes; base->codes and
 * resid_full are not read (they may be NULL).
 * Then blocks are ordered by (Delta descending, b ascending): rank[0..budget) = the
 * first `budget` indices in that order, sel[0..budget) = the same set ascending.
 * delta: fp64 [(N/64)*(K/64)]. 0 <= budget <= number of blocks.
 * ws: mq_delta_topk_workspace_bytes.
 */
mq_status mq_delta_score_topk(const mq_bf16* W, const float* H, const mq_nvfp4_mat* base,
                              const mq_nvfp4_mat* resid_full, int budget, double* delta, int32_t* rank,
                              int32_t* sel, void* ws, size_t ws_bytes, mq_stream stream);

/*
 * A1 + A3 in one pass over W (same results as mq_quantize_weight followed by the
 * Delta part of mq_delta_score_topk): base NVFP4 codes and scales, the tensor scale,
 * Delta [(N/64)*(K/64)] (fp64) with H from mq_hessian_diag, and, if resid_full is not
 * NULL, the full residual's codes and sf. resid_full == NULL skips storing the residual
 * (mq_pack_residual_weight recomputes the selected blocks from W). base->sf may be NULL.
 * W is read before the call waits for the preceding kernel in the stream (it must not be
 * written by a kernel that lets its dependents start early). Buffers and workspace as in
 * mq_quantize_weight; base->codes and sf_swz 16-byte aligned.
 */
mq_status mq_quantize_weight_delta(const mq_bf16* W, int N, int K, const float* H, mq_nvfp4_mat* base,
                                   mq_nvfp4_mat* resid_full, double* delta, void* ws, size_t ws_bytes,
                                   mq_stream stream);

/*
 * A4 alone: order nblk blocks by (Delta descending, block index ascending); rank gets the
 * first `budget` indices in that order, sel the same set ascending. 0 <= budget <= nblk.
 */
mq_status mq_topk_blocks(const double* delta, int nblk, int budget, int32_t* rank, int32_t* sel, mq_stream stream);

/*
 * A5. Pack the selected residual blocks (the sparse residual of section 1, stored per
 * block for the fused GEMM's "sparse block computation", arXiv abstract).
 * resid_full: codes and sf of mq_quantize_weight. sel: ascending block indices [budget].
 * out: N, K, nblk = budget, and buffers sized as in mq_residual_packed.
 */
mq_status mq_pack_residual(const mq_nvfp4_mat* resid_full, const int32_t* sel, int budget,
                           mq_residual_packed* out, mq_stream stream);

/*
 * A5 straight from W: the selected blocks' residual is recomputed with the weight
 * quantizer's arithmetic (base group, R = W - deq Q(W), NVFP4(R) with the tensor scale
 * base->gscale) and written packed; the result is bit-identical to mq_pack_residual on
 * mq_quantize_weight's resid_full, and the full residual never has to be stored.
 * W: bf16 [N][K] (16-byte aligned). base: rows = N, cols = K, gscale (from
 * mq_quantize_weight or mq_quantize_weight_delta); its codes are not read.
 * sel: ascending block indices [budget]. out: as in mq_pack_residual.
 */
mq_status mq_pack_residual_weight(const mq_bf16* W, const mq_nvfp4_mat* base, const int32_t* sel, int budget,
                                  mq_residual_packed* out, mq_stream stream);

/*
 * A6. Activation quantization (summary, "Methodology", section 3: quantization inside
 * the pipeline). X: bf16 [M][K]. Per token m: g_x[m] = amax(X[m,:]) / 2688 (1 if 0),
 * then NVFP4 with that scale. xq: codes, sf_swz and gscale[M] required, sf optional.
 * K <= 65536 (MQ_ERR_UNSUPPORTED_SHAPE above). X 16-byte aligned, codes 8, sf_swz 4.
 */
mq_status mq_quantize_act(const mq_bf16* X, int M, int K, mq_nvfp4_mat* xq, mq_stream stream);

/*
 * A7 + A8. ZipperEngine fused GEMM (summary, "Methodology", section 3; arXiv abstract):
 *   Y[m,n] = bf16_rn( acc[m,n] * fp32(g_x[m] * g_w) ),
 *   acc[m,n] = sum_k xh[m,k] * ( wh[n,k] + [block (n/64, k/64) selected] rh[n,k] ),
 * with xh, wh, rh the scaled E2M1 values (val * dec(sf)). Base and residual blocks
 * accumulate into one fp32 tensor-memory accumulator (tcgen05 kind::mxf4nvf4 MMAs, one
 * extra MMA per selected block). The decode kernel (small M) gives every SM an equal
 * share of the (tile, 256-K) work units; a tile whose K range is split between CTAs is
 * summed from their fp32 partials in a fixed order, so repeated calls give the same bits.
 * r == NULL (or r->nblk == 0) is the dense base alone.
 * xq: codes, sf_swz, gscale [M]. wq: codes, sf_swz, gscale [1]. Y: bf16 [M][N].
 * flags: MQ_GEMM_* (one of AUTO/DECODE/PREFILL, optionally BASE_ONLY or RESIDUAL_ONLY).
 * MQ_GEMM_WEIGHTS_READY: the caller guarantees that no kernel that may still be running
 * when this call's kernel starts writes wq or r (as for a layer's weights at inference,
 * prepared once); the decode kernel then requests its first W stages before it waits for
 * the preceding kernel in the stream, so they overlap that kernel's tail. X, g_x, Y and
 * the workspace are still touched only after that wait. Without the flag every input is
 * read after the wait.
 * ws: mq_gemm_workspace_bytes(M, N, K, flags) bytes (see there); may be NULL if that
 * size is 0.
 */
mq_status mq_gemm(const mq_nvfp4_mat* xq, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y,
                  int M, int N, int K, unsigned flags, void* ws, size_t ws_bytes, mq_stream stream);

/*
 * A6 + A7 + A8 in one kernel: the activation quantization runs inside the fused GEMM's
 * pipeline ("quantization ... scheduled concurrently" with the dense and sparse MMAs and
 * the reduce-sum: summary, "Methodology", section 3), for the decode kernel. X: bf16
 * [M][K] (16-byte aligned). Each CTA quantizes the tokens of its tile over its K range
 * straight into the MMA's operand layout; the per-token scale g_x[m] = amax(X[m,:])/2688
 * (1 if 0) comes from maxima exchanged between the K splits of a tile through the
 * thread-block cluster's shared memory (or, for more than 8 splits, each CTA reads the
 * whole row). The codes and scales are those of mq_quantize_act (bit-identical); this
 * kernel splits K at fixed points of its own, so Y equals mq_gemm's within the GEMM's
 * tolerance, not bit for bit. gx_out: [M] fp32, receives g_x, or NULL. Other
 * arguments, flags and workspace as in mq_gemm; MQ_GEMM_PREFILL returns
 * MQ_ERR_UNSUPPORTED_SHAPE (the large-M kernel takes a quantized X).
 */
mq_status mq_gemm_act(const mq_bf16* X, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y, int M, int N,
                      int K, unsigned flags, void* ws, size_t ws_bytes, float* gx_out, mq_stream stream);

/*
 * Device buffers of one layer for mq_run_layer (all caller-owned; sizes as in the
 * individual calls above). W_dev, X_dev, Xcal_dev and Y_dev are staging buffers used
 * only when mq_run_layer is given host pointers.
 */
typedef struct {
    mq_nvfp4_mat base;        /* sf may be NULL */
    mq_nvfp4_mat resid_full;  /* not used by mq_run_layer (may be all zero) */
    mq_nvfp4_mat xq;          /* codes, sf_swz, gscale [M] */
    float* H;                 /* [K] */
    double* delta;            /* [(N/64)*(K/64)] */
    int32_t* rank;            /* [budget] */
    int32_t* sel;             /* [budget] */
    mq_residual_packed packed;
    void* ws_quant;           /* mq_quantize_weight_workspace_bytes */
    size_t ws_quant_bytes;
    void* ws_gemm;            /* mq_gemm_workspace_bytes (counters zeroed once) */
    size_t ws_gemm_bytes;
    mq_bf16* W_dev;           /* [N][K]  staging when host != 0 */
    mq_bf16* X_dev;           /* [M][K]  staging when host != 0 */
    mq_bf16* Xcal_dev;        /* [T][K]  staging when host != 0 */
    mq_bf16* Y_dev;           /* [M][N]  staging when host != 0 */
} mq_layer_buffers;

/*
 * The whole path for one layer: A2 H from the T calibration tokens, A1+A3 quantize W and
 * score every block (mq_quantize_weight_delta, residual not stored), A6 quantize X
 * (mq_quantize_act's results; for K <= 4096 the quantize+Delta kernel's least loaded CTAs
 * quantize the rows after their strips, otherwise its own kernel runs ahead of the
 * selection), A4 top-`budget` selection, A5 pack the selected residual from
 * W (mq_pack_residual_weight), A7+A8 fused GEMM into Y. Results are those of the
 * individual calls. The call's first kernel waits for the kernel preceding the call in
 * the stream before the others may start, so no input is read before that kernel ends.
 * With host == 0, W, X, Xcal and Y are device pointers. With host != 0 they are HOST
 * pointers (page-locked for the copies to be asynchronous): the inputs are copied into
 * buf->W_dev, X_dev, Xcal_dev and the result from buf->Y_dev back to Y, all on `stream`.
 * flags: the GEMM flags, plus MQ_LAYER_PREPARED for inference on a layer whose weight a
 * previous call prepared: buf->base and buf->packed already hold the quantized weight and
 * the packed residual of `budget` blocks, A1..A5 are skipped, W and Xcal are not read
 * (they may be NULL) and only X (and Y) cross the host link. Errors as the individual
 * calls.
 */
mq_status mq_run_layer(const mq_bf16* W, const mq_bf16* X, const mq_bf16* Xcal, mq_bf16* Y, int M, int N, int K,
                       int T, int budget, unsigned flags, int host, mq_layer_buffers* buf, mq_stream stream);

/*
 * mq_gemm without a workspace argument, for callers that cannot allocate device memory
 * (for example code embedded in a framework that owns all device memory and offers no
 * workspace hook, or paths where an allocation is not allowed). The paper has no
 * counterpart to this call; it exists for such integrations.
 * Same arguments, checks, kernel choice (the flags, else by shape) and results as
 * mq_gemm, minus ws/ws_bytes. The decode kernel's scratch (fp32 partials of the tiles
 * that CTAs share, and the tile counters) is a static array inside the library,
 * mq_gemm_noalloc_scratch_limit() bytes (16 MiB) on every GPU that loads the library,
 * held until the process exits; the large-M kernel needs none. A problem whose
 * mq_gemm_workspace_bytes() exceeds that limit (decode shapes with more than 64 tokens)
 * is rejected with MQ_ERR_WORKSPACE before anything is launched (use mq_gemm with a
 * workspace instead). The first call on each device looks up the
 * array's device address (set-up, once per device, with that device current); make
 * that first call before any stream capture. Each call clears the scratch's tile
 * counters on `stream` before its kernel. All calls share the one array, which keeps
 * the last call's contents: calls that overlap on the GPU race and must be serialized
 * by the caller. Allocates nothing (no cudaMalloc/cudaFree).
 */
mq_status mq_gemm_noalloc(const mq_nvfp4_mat* xq, const mq_nvfp4_mat* wq, const mq_residual_packed* r, mq_bf16* Y,
                          int M, int N, int K, unsigned flags, mq_stream stream);

/* Size in bytes of mq_gemm_noalloc's static scratch array. */
size_t mq_gemm_noalloc_scratch_limit(void);

/* Synchronizes `stream`, then returns (and clears) the device error word: MQ_OK, or
 * MQ_ERR_TIMEOUT if a kernel gave up on a pipeline wait, or MQ_ERR_CUDA if the
 * synchronization itself failed. */
mq_status mq_get_error(mq_stream stream);

/* Static description of a status code. */
const char* mq_status_string(mq_status status);

/* Number of kernel launches the library has issued in this process (for accounting). */
uint64_t mq_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOSAIC_H_ */

/*
 * mosaic_probe.h -- measurement helper of libmosaic (not a step of the path).
 *
 * The dense FP4 tensor-core rate that the fused GEMM's large-M kernel is compared with,
 * measured on the GPU at hand rather than taken from a datasheet. The pages time their
 * kernel on other hardware and print no tensor-core figure; this has no counterpart
 * there.
 */
#ifndef MOSAIC_PROBE_H_
#define MOSAIC_PROBE_H_

#include "mosaic.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Launches `ctas` CTAs (one per SM gives the whole GPU) on `stream`. Each keeps a
 * 128 x 256-K E2M1 A tile, a 256 x 256-K B tile and their E4M3 scales (all 1.0)
 * resident in shared and tensor memory and issues `iters` back-to-back
 * tcgen05.mma.kind::mxf4nvf4.block_scale (M = 128, N = 256, K = 64) into one fp32
 * accumulator, with no memory traffic in the loop. Time it with events on `stream`;
 * mq_fp4_mma_loop_flops(ctas, iters) is the work done. Allocates nothing. Returns
 * MQ_ERR_INVALID_ARG unless ctas >= 1 and 1 <= iters <= 2^24, MQ_ERR_CUDA if the launch
 * fails; a final wait that gave up (2 s) is reported by mq_get_error.
 */
mq_status mq_fp4_mma_loop(int ctas, int iters, mq_stream stream);

/* 2 * 128 * 256 * 64 flops per MMA, times ctas * iters. */
double mq_fp4_mma_loop_flops(int ctas, int iters);

/*
 * Event times of the small-problem decode GEMM (the cluster-split kernel), for a library
 * built with MQ_TIMELINE defined (bit_quantized_gemm_zipperengine_b200/build.py builds it as
 * libmosaic_timeline.so): every launch records %globaltimer (ns) at fixed points of its
 * first MQ_TIMELINE_CTAS CTAs, over the previous launch's values. The table is
 * uint64 [MQ_TIMELINE_CTAS][MQ_TIMELINE_EVENTS], 0 where an event did not happen:
 *   0 CTA set up (barriers initialised, tensor memory allocated)
 *   1 first W copies issued          2 the wait for the preceding kernel returned
 *   3 first X copies issued          4 first stage landed (MMA issuer)
 *   5 last MMAs issued               6 accumulator complete (epilogue)
 *   7 partial in shared memory, first cluster barrier passed
 *   8 this CTA's rows added and stored   9 last cluster barrier passed
 * Copies the table into `out` (host memory of at least `bytes` >= its size) and clears
 * it on the device. Synchronous with the device. Returns MQ_ERR_INVALID_ARG for a null
 * or short `out`, and in a library built without MQ_TIMELINE; MQ_ERR_CUDA if a copy
 * fails.
 */
#define MQ_TIMELINE_CTAS 160
#define MQ_TIMELINE_EVENTS 16
mq_status mq_timeline_read(void* out, size_t bytes);

#ifdef __cplusplus
}
#endif

#endif /* MOSAIC_PROBE_H_ */

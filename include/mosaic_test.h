/*
 * mosaic_test.h -- test hook of libmosaic (not a step of the path).
 *
 * Every pipeline wait in the library's kernels is bounded: a wait that runs out records
 * MQ_ERR_TIMEOUT in the device error word, the kernel stops issuing work, releases its
 * tensor memory and returns, and mq_get_error() reports the status on the host. This
 * hook lets a test make one such wait run out on purpose, without faulting anything.
 * The pages have no counterpart to it.
 */
#ifndef MOSAIC_TEST_H_
#define MOSAIC_TEST_H_

#include "mosaic.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Arms the next decode-kernel launch of mq_gemm / mq_gemm_noalloc in this process (one
 * launch, then the hook disarms itself; either decode kernel, the small-problem one or
 * the stream-K one): CTA 0 never requests the W tile of its `unit`-th work unit (unit >= 0;
 * no effect if the CTA has fewer units), and every pipeline wait of that launch gives up
 * after wait_ms milliseconds (0.01 <= wait_ms <= 2000) instead of 2 s.
 * The MMA issuer's wait for that stage then runs out with no copy in flight for it; the
 * launch ends with MQ_ERR_TIMEOUT in the device error word (read it with mq_get_error),
 * its output is incomplete, and the workspace's tile counters may be left non-zero (zero
 * them before the workspace's next call). MQ_ERR_INVALID_ARG for arguments out of range.
 */
mq_status mq_test_arm_wait_fault(int unit, double wait_ms);

#ifdef __cplusplus
}
#endif

#endif /* MOSAIC_TEST_H_ */

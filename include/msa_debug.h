/* msa_debug.h -- instrumentation and test hooks of libmsa (not part of the
 * Memory Sparse Attention path; the product calls are in msa.h).
 *
 * They let a benchmark time the routing scan inside a step, and let tests
 * drive the library's failure paths without a device fault: a host-to-device
 * copy made to fail before it reaches the GPU, and an in-kernel wait made to
 * run out. */
#ifndef MSA_DEBUG_H
#define MSA_DEBUG_H

#include "msa.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Every in-kernel wait (on an mbarrier of a copy or a pipeline stage) is
 * bounded: after limit_us of wall time (1 s in the kernels) it gives up,
 * sets MSA_DEV_PIPE_TIMEOUT and lets the kernel finish, so that the context
 * stays usable.  This diagnostic runs that path on purpose: 64 threads wait
 * on a barrier nothing arrives at, with the given limit (0: the kernels' own
 * limit).  Writes how many threads gave up (all 64 when the path works) and
 * blocks until done; the status bit is then set. */
msa_status msa_debug_expire_wait(int64_t limit_us, int32_t* lanes_gave_up, cudaStream_t stream);

/* ------------------------------------------------------ instrumentation */

/* When both events are non-NULL, every later msa_route / msa_route_scores
 * call on the calling thread records `start` immediately before and `stop`
 * immediately after its router-key scan kernel, on that call's stream, so the
 * scan's duration can be read with cudaEventElapsedTime.  NULL, NULL turns it
 * off.  Used by the benchmark to time the dominant kernel inside a step. */
void msa_debug_scan_events(cudaEvent_t start, cudaEvent_t stop);

/* ------------------------------------------------------------ test hook */

/* Makes the next n host-to-device copies issued by msa_fetch_selected on the
 * calling thread fail with MSA_ERR_CUDA without reaching the GPU, so that
 * error paths can be tested without a device fault.  n = 0 disarms it. */
void msa_debug_fail_next_copies(int32_t n);

#ifdef __cplusplus
}
#endif
#endif /* MSA_DEBUG_H */

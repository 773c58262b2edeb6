/*
 * mnb_tune.h -- tuning hooks of libmnb.so, for sweeps of the kernels' launch
 * shapes.  Not part of the stable ABI of mnb.h: they change process-wide state
 * that every later call on every thread sees, and exist so that a measurement
 * script can force a tile or split choice without rebuilding the library.
 * Each returns MNB_OK, or MNB_ERR_INVALID_ARG for an argument outside its range
 * (and then changes nothing).
 */
#ifndef MNB_TUNE_H
#define MNB_TUNE_H

#include "mnb.h"

#ifdef __cplusplus
extern "C" {
#endif

/* mnb_gemm: smallest token tile (16..256, a multiple of 16) the tile heuristic
 * may choose, and the largest cluster split of K (1..8).  Defaults 128 and 4. */
MNB_API int mnb_tune_gemm(int min_bn, int max_split);

/* mnb_gemm: smallest and largest token tile (16 <= min_bn <= max_bn <= 256)
 * and the largest cluster split of K (1..8). */
MNB_API int mnb_tune_gemm_tiles(int min_bn, int max_bn, int max_split);

/* fp16 decode GEMV (mnb_gemv, mnb_gemv_swiglu): force the K split to w warps
 * (1, 2, 4 or 8) x s clustered CTAs (1..8) per 16-row tile; w = 0 gives the
 * choice back to the planner. */
MNB_API int mnb_tune_gemv_split(int w, int s);

/* fp16 decode GEMV at M = 1: 1 (default) runs the kernel whose CTAs hold
 * their whole share of the weights in shared memory, where the shape allows
 * it; 0 runs the general decode kernel. */
MNB_API int mnb_tune_gemv_resident(int enable);

/* Fault injection for tests of mnb_gemv_chain's timeout path (no GPU fault,
 * no hang): every later launch leaves task `task` uncounted, so the next task
 * that waits for it gives up after wait_limit_us microseconds (0 = the
 * default 2 s), sets status bit 2 and the workspace's abort word, and exits.
 * task = -1 turns the injection off; the last task's count is never withheld.
 * wait_limit_us <= 2000000. */
MNB_API int mnb_test_chain_withhold(int task, int wait_limit_us);

#ifdef __cplusplus
}
#endif

#endif /* MNB_TUNE_H */

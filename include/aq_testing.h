/*
 * aq_testing.h — test hooks of libaq (not for production use).
 *
 * They let a test drive the failure path of the decode kernels' bounded waits
 * (the bound every mbarrier wait of a kernel has, after which the kernel stops
 * issuing work, lets its copies in flight land, sets bit 0 of
 * aq_device_errors() and returns) without faulting the GPU: the host shortens
 * the bound and delays one role of the kernel past it, so that the waits of
 * the other roles run out.  The pages have no counterpart.
 *
 * Scope: the warp-MMA decode kernel behind aq_qmv / aq_qmv_batched /
 * aq_qmv_noalloc (4-bit affine weights), aq_qmv's kernel choice, and
 * aq_gather_qmm's grouping of index pairs.  The
 * settings are process-wide and apply to launches made after the call; 0
 * restores the default.
 */
#ifndef AQ_TESTING_H
#define AQ_TESTING_H

#include "aq.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bound of every mbarrier wait of the decode kernel, in ns (default 2 s). */
AQ_API void aq_testing_set_wait_limit_ns(uint64_t ns);

/* Delay, in ns, before the decode kernel's TMA warp issues its first copy
 * (default 0).  The delay ends early once another role has given up. */
AQ_API void aq_testing_set_start_delay_ns(uint64_t ns);

/* Kernel that later aq_qmv calls of this process use where it applies:
 * 0 the automatic choice (default), 1 the warp-MMA decode kernel, 2 the
 * tcgen05 decode kernel, 3 the fp32 CUDA-core kernel (any other value:
 * automatic).  Lets a test run each
 * kernel on the same shapes; the workspace that aq_workspace_size reports
 * covers every kernel. */
AQ_API void aq_testing_set_qmv_kernel(int which);

/* The expert grouping aq_gather_qmm would use for these index pairs (host
 * logic only, no launch): returns the number of grouped problems (0 when the
 * pairs run ungrouped) and writes the rows per problem and, for up to
 * map_rows rows, the row maps: xmap[r] = the row of x (viewed as
 * [x_batch * M, K]) that problem row r reads, ymap[r] = the row of y (viewed
 * as [n_pairs * M, N]) it writes; -1 marks a padding row. */
AQ_API int aq_testing_gather_groups(const int32_t* lhs_indices, const int32_t* rhs_indices,
                                    int64_t n_pairs, int64_t M, int64_t N, int64_t K,
                                    int64_t x_batch, int32_t* xmap, int32_t* ymap,
                                    int64_t map_rows, int* rows_per_group);

/* Clears the device error bits that aq_device_errors() reports.  Synchronises
 * the current device first. */
AQ_API aq_status aq_testing_clear_device_errors(void);

#ifdef __cplusplus
}
#endif

#endif

/*
 * tidar_testing.h -- test hooks of the TiDAR decode-step library.  Not part of
 * the decode path: nothing in a decode step calls these.
 *
 * The paper has no counterpart to these calls: they exist so that the failure
 * handling documented in tidar.h ("no kernel traps, asserts or waits without a
 * bound") can be exercised on a GPU without faulting or hanging it.
 */
#ifndef TIDAR_TESTING_H
#define TIDAR_TESTING_H

#include "tidar.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * tidar_attn_step with a wait that runs out on purpose.  Arguments as in
 * tidar_attn_step (no workspace), plus:
 *
 * wait_cycles  bound of every on-chip wait of the launch, in SM clock cycles
 *              (tidar_attn_step uses about 2 s worth); must be >= 1.
 *
 * Before its first MMA the kernel's MMA-issuing thread waits on a barrier
 * nothing ever arrives on.  That wait runs out after wait_cycles; the kernel
 * then stops every role, waits for the copies and MMAs it already issued,
 * frees its tensor memory, sets TIDAR_DEV_TIMEOUT in *dev_status and returns:
 * the context stays usable.  The outputs are not valid.  Other status codes
 * as tidar_attn_step.
 */
tidar_status tidar_testing_attn_step_stalled(const void *q, const void *k_new, const void *v_new,
                                             const void *k_cache, const void *v_cache, const int32_t *prefix_len,
                                             int B, int Hq, int Hkv, int D, int k, int P_max,
                                             float softmax_scale, int mask_mode, void *out, float *lse,
                                             int32_t *dev_status, long long wait_cycles, void *stream);

/*
 * The cluster size (key splits per row tile) tidar_attn_step would use for
 * these sizes on the current device (the largest that keeps every row tile's
 * cluster resident in one wave; 1 when even single CTAs need several waves),
 * or 0 for sizes tidar_attn_step rejects.  Queries the device's cluster
 * occupancy; launches nothing.
 */
int tidar_testing_attn_splits(int B, int Hq, int Hkv, int D, int k, int P_max);

#ifdef __cplusplus
}
#endif
#endif /* TIDAR_TESTING_H */

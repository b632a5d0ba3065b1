/*
 * kata_profile.h — kernel timing instrumentation of libkata.
 *
 * The paper has no counterpart: this exists so that benchmarks can time each
 * kernel of a forward or decode call live, with CUDA events recorded on the
 * call's own stream around every kernel launch.  Off by default; when off,
 * the entry points of kata.h record nothing.  Not thread-safe against
 * concurrent kata_* calls from other host threads while enabled.
 */
#ifndef KATA_PROFILE_H_
#define KATA_PROFILE_H_

#include "kata.h"

#ifdef __cplusplus
extern "C" {
#endif

/* enable != 0: start recording (and drop earlier records); 0: stop.
 * At most 65536 launches are recorded; later launches are counted in
 * kata_profile_dropped() but not timed. */
kata_status kata_profile_enable(int enable);

/* Waits for every recorded launch to finish, then returns the number of
 * distinct kernels recorded so far (or -1 on a CUDA error). */
int kata_profile_kernel_count(void);

/* For kernel idx in [0, kata_profile_kernel_count()): its name (static
 * string owned by the library), number of launches, and the sum of their
 * durations in milliseconds. */
kata_status kata_profile_kernel(int idx, const char **name, int *launches, double *total_ms);

/* Launches not timed because the record limit was reached. */
int kata_profile_dropped(void);

#ifdef __cplusplus
}
#endif

#endif /* KATA_PROFILE_H_ */

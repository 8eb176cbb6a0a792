/*
 * msda_checked.h -- extra entry points of the bounds-checked build of the
 * library, libmsda_checked.so.
 *
 * libmsda_checked.so is compiled from the same sources as libmsda.so with
 * -DMSDA_CHECKED and exports every function of msda.h and msda_debug.h plus
 * the two below.  It is a debugging build, standing in for a race and
 * bounds sanitizer:
 *
 *  - Every gather of a value row chunk and every vector reduction into
 *    grad_value first tests its element range [first, first + count) against
 *    the value map [0, limit), limit = N*S*M*D by default.  An access outside
 *    it is not made: a gather reads zeros instead, a scatter is dropped.  The
 *    kernel counts such accesses in a device word and records the element
 *    index of the first one.  Nothing traps, asserts or faults.
 *  - After its launch, each compute entry point waits for `stream` (the only
 *    synchronising path of either build), reads the word, clears it, and
 *    returns MSDA_ERR_DEVICE_CHECK if it counted anything.  The outputs are
 *    then those of the computation with the skipped accesses reading zero.
 *  - The device word is one per device, shared by all streams and threads:
 *    calls that overlap in time on one device (two streams, two host threads)
 *    may see each other's violations.  Serialise calls when checking.
 *
 * The checks cost registers and instructions; the kernels of this build are
 * not the ones to time.
 */
#ifndef MSDA_CHECKED_H
#define MSDA_CHECKED_H

#include <stdint.h>

#include "msda.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Lower the bound that the checks test against: value_elements >= 0 makes
 * every later call use min(value_elements, N*S*M*D) as the limit; a negative
 * value restores the default N*S*M*D.  Process-wide; takes effect for calls
 * made after it returns.  This lets a test make the checks fire on valid
 * inputs (accesses at or beyond the lowered bound are skipped and reported)
 * while every access that is made stays inside the caller's buffers.
 * Returns MSDA_OK.
 */
MSDA_API msda_status msda_checked_set_limit(int64_t value_elements);

/*
 * The calling thread's last MSDA_ERR_DEVICE_CHECK: *count = accesses skipped
 * in that call, *first_element = the element index (into the [N,S,M,D] value
 * map and grad_value) of the first one recorded.  Both 0 / -1 when the thread
 * has seen no violation.  Either pointer may be NULL.
 * Returns MSDA_OK.
 */
MSDA_API msda_status msda_checked_last_violation(int64_t *count, int64_t *first_element);

#ifdef __cplusplus
}
#endif

#endif /* MSDA_CHECKED_H */

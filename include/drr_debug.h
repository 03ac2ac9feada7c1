/*
 * drr_debug.h -- the bounds-checked debug build of libdrr (libdrr_checked.so).
 *
 * The same sources compiled with -DDRR_BOUNDS_CHECK: every gather and
 * scatter of every kernel (volume reads of every layout, image reads and
 * writes, gradient-volume, corner-record and pose-gradient atomics, the
 * prepare passes' reads) tests its element range against the extent of the
 * buffer, or of the volume-channel slot, it addresses.  An access outside is
 * skipped (a load reads 0) and counted in a device error word.  The checked
 * library exports every entry point of drr.h, with the same arguments and
 * results as long as no access is out of range, plus the call below; the
 * ordinary libdrr.so does not export it.
 */
#ifndef DRR_DEBUG_H
#define DRR_DEBUG_H

#include "drr.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Out-of-range accesses counted since the last call, over every kernel of
 * the library on the current device (*count), and the element offset of one
 * of them (*first; 0 when *count is 0); both words are cleared.  Reads
 * device memory synchronously: call it after the work has completed (the
 * stream synchronised).  Returns DRR_OK, DRR_ERR_INVALID_ARG for NULL
 * pointers, or DRR_ERR_CUDA if a copy fails. */
DRR_API drr_status drr_debug_bounds_errors(unsigned long long *count, long long *first);

#ifdef __cplusplus
}
#endif

#endif /* DRR_DEBUG_H */

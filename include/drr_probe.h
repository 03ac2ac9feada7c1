/*
 * drr_probe.h -- measurement helpers of the benchmark (libdrr_probe.so), not
 * part of the ray-march.  They measure the L2 read bandwidth that is the
 * denominator of the gather roofline while a volume fits in L2 (the
 * measured-peaks file of the GPU pool has HBM and GEMM peaks only), and the
 * L2's fp32 reduction throughput, the ceiling of the adjoint's scatter.
 */
#ifndef DRR_PROBE_H
#define DRR_PROBE_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DRR_PROBE_API __attribute__((visibility("default")))
#else
#define DRR_PROBE_API
#endif

/* Streams `reps` passes of float4 reads over the DEVICE buffer `buf`
 * (n_vec16 16-byte vectors, 16-byte aligned) with loads that bypass L1
 * (ld.global.cg), so a buffer that fits in L2 is read from L2.  Writes one
 * float to the DEVICE word `sink` only if the sum is NaN (never, for finite
 * data) so the loads cannot be optimised away.  Asynchronous on `stream`
 * (a cudaStream_t).  Returns 0, or -1 for bad arguments (nothing launched),
 * or the CUDA error code of a failed launch.  Bytes read: n_vec16 * 16 * reps. */
DRR_PROBE_API int drr_probe_l2_read(const void *buf, size_t n_vec16, int reps, float *sink,
                                    void *stream);

/* fp32 atomic reductions (red.global.add) over the DEVICE buffer `buf`
 * (n_floats floats, a multiple of 8, 32-byte aligned; it should fit in L2),
 * `reps` passes, each adding 1.0f to the floats its pattern touches:
 *   kind 0  scalar reductions, a warp on 32 consecutive floats: every float
 *           once per pass, n_floats / 8 sector operations of 8 values;
 *   kind 1  16-byte vector reductions, two per 32-byte record: every float
 *           once per pass, n_floats / 4 sector operations of 4 values;
 *   kind 2  one scalar reduction on the first float of each 32-byte sector:
 *           n_floats / 8 sector operations of 1 value.
 * The buffer's contents change (the caller zeroes it if it cares).
 * Asynchronous on `stream`.  Returns 0, -1 for bad arguments (nothing
 * launched), or the CUDA error code of a failed launch. */
DRR_PROBE_API int drr_probe_l2_red(float *buf, size_t n_floats, int reps, int kind,
                                   void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DRR_PROBE_H */

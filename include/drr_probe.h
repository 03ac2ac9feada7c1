/*
 * drr_probe.h -- measurement and self-test helpers (libdrr_probe.so), not
 * part of the ray-march.  They measure the L2 read bandwidth that is the
 * denominator of the gather roofline while a volume fits in L2 (the
 * measured peak figures at hand cover HBM and GEMMs only), and the
 * L2's fp32 reduction throughput, the ceiling of the adjoint's scatter; and
 * they drive the adjoint's grid barrier, including a wait that runs out.
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

/* Self-test of the bounded grid barrier that separates the phases of the
 * volume adjoint's slab pass (drr_render_adjoint_ws): one CTA per SM,
 * launched cooperatively, passes `rounds` barriers, each expecting the
 * grid's CTA count plus `extra_arrivals`.  With extra_arrivals = 0 every
 * barrier completes; with more, no epoch completes, the first wait that
 * lasts timeout_ms raises the abort word and every CTA returns.  Reports the
 * waits that gave up (*timeouts_out), the barriers passed summed over CTAs
 * (*passes_out) and the CTA count (*ctas_out).  Synchronous (allocates and
 * frees a few words, synchronises the device).  Returns 0, -1 for bad
 * arguments (rounds in [1, 4096], timeout_ms in (0, 60000]), or a CUDA
 * error code. */
DRR_PROBE_API int drr_probe_grid_barrier(int extra_arrivals, int rounds, double timeout_ms,
                                         unsigned long long *timeouts_out, int *passes_out,
                                         int *ctas_out);

#ifdef __cplusplus
}
#endif

#endif /* DRR_PROBE_H */

/*
 * drr_probe.h -- measurement helper of the benchmark (libdrr_probe.so), not
 * part of the ray-march.  It measures the L2 read bandwidth that is the
 * denominator of the gather roofline while a volume fits in L2 (the
 * measured-peaks file of the GPU pool has HBM and GEMM peaks only).
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

#ifdef __cplusplus
}
#endif

#endif /* DRR_PROBE_H */

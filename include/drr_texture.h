/*
 * drr_texture.h -- the texture-trilinear comparison (libdrr_texture.so).
 *
 * NOT the product path: a measured comparison of the forward ray-march in
 * which the GPU's texture units do the trilinear interpolation (hardware
 * filtering, whose interpolation weights are 8-bit fixed point: TorchTomo
 * page, "Fast CUDA Kernels": texture sampling is fast but about 1e-4
 * relative from the exact forward).  It is kept to measure that trade
 * against the exact kernels of libdrr.so, and is accepted only where its
 * error meets the parity tolerance.
 *
 * Same geometry, sample placement, modes and image layout as drr_render
 * (include/drr.h).  Unlike libdrr.so this library allocates: the texture
 * needs a CUDA 3-D array, made by drr_tex_create and released by
 * drr_tex_destroy.  Return values: 0 on success, -1 for invalid arguments
 * (nothing done), otherwise the CUDA error code; drr_tex_last_error()
 * describes the last failure of this thread.
 */
#ifndef DRR_TEXTURE_H
#define DRR_TEXTURE_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DRR_TEX_API __attribute__((visibility("default")))
#else
#define DRR_TEX_API
#endif

typedef struct drr_tex_volume drr_tex_volume;   /* opaque */

/* Copy a DEVICE float32 volume vol[k][j][i] (dims {nx, ny, nz}, each >= 2)
 * into a 3-D texture with zero border and linear filtering.  texel: 0 =
 * float32 texels, 1 = float16 texels (rounded to nearest).  Synchronous
 * (returns when the texture is ready).  *out receives the handle. */
DRR_TEX_API int drr_tex_create(const float *vol, const int dims[3], int texel,
                               drr_tex_volume **out);

/* Forward projection through the texture: arguments as drr_render
 * (include/drr.h) for the geometry, modes and output; asynchronous on
 * `stream` (a cudaStream_t). */
DRR_TEX_API int drr_tex_render(const drr_tex_volume *tex, const float spacing[3],
                               const float origin[3], const float K[9], const float *Rt, int B,
                               int H, int W, int n_samples, float density_factor, int mode,
                               float *out, void *stream);

/* Release the texture and its array (synchronises the device first). */
DRR_TEX_API int drr_tex_destroy(drr_tex_volume *tex);

DRR_TEX_API const char *drr_tex_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DRR_TEXTURE_H */

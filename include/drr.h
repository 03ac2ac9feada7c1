/*
 * drr.h -- C ABI of the B200 cone-beam DRR ray-marcher (libdrr.so).
 *
 * What the library computes (all entry points follow the same geometry):
 *
 *   A digitally reconstructed radiograph of a 3-D attenuation volume seen by
 *   a pinhole camera.  For every detector pixel of every view, a ray leaves
 *   the source through the pixel centre (Hartley-Zisserman camera
 *   x ~ K [R | t] X: nanodrr page, introduction), is clipped to the volume
 *   box with the slab method (flashdrr.rendering API docs,
 *   VolumeRaycaster.compute_clipping_distances: near/far from the volume
 *   bounds), is sampled n_samples times uniformly with zero-padded trilinear
 *   interpolation in IJK voxel space (VolumeRaycaster.forward: the volume
 *   lives in IJK space, an affine maps world to IJK; VolumeRaycaster.__init__:
 *   ray_samples), and yields I = density_factor * sum(mu * dt)
 *   (VolumeRaycaster.__init__: density_factor), written raw or as the
 *   Beer-Lambert image 1 - exp(-I) (VolumeRaycaster.__init__:
 *   use_beer_lambert).  The adjoint scatters an image-space gradient back
 *   along the same rays (TorchTomo page, "Discrete Adjoint and Learned
 *   Primal-Dual": <A x, y> = <x, A^T y>; FlashDRR page, "Train vs. Eval
 *   Dynamics": backward gradient kernels of the fused renderer).
 *
 * Conventions shared by every entry point
 *
 *   volume    vol[k][j][i], i fastest; dims = {nx, ny, nz}, each >= 2.
 *             World position of voxel (i, j, k) = origin + spacing * (i, j, k):
 *             origin (mm) is the CENTRE of voxel 0, spacing (mm) > 0.
 *   box       rays are clipped to the box spanned by the voxel centres,
 *             [0, n-1] per axis in IJK.  Samples: midpoint rule,
 *             dt = (t1 - t0) / n_samples, t_i = t0 + (i + 1/2) dt, with
 *             t0 = max(t_near, 0), t1 = t_far in world mm along the unit
 *             ray; t1 <= t0 is a miss and gives I = 0.
 *   camera    K: HOST array, 9 floats row-major, upper triangular
 *             [fx s cx; 0 fy cy; 0 0 k22], fx, fy, k22 non-zero.
 *             Rt: DEVICE array, B x 12 floats, row-major [R | t] per view,
 *             world -> camera, R a rotation.  Pixel (row r, col c) has its
 *             centre at (u, v) = (c, r); camera +z looks into the scene.
 *   images    out / grad_out / fwd_out: DEVICE, float32 [B][H][W].
 *   stream    a cudaStream_t passed as void* (NULL = legacy default stream).
 *
 * Ownership and semantics: the caller owns every buffer.  The library keeps
 * no state between calls and allocates no device memory.  Host arrays
 * (dims, spacing, origin, K) are read during the call only.  Every call is
 * asynchronous on `stream`; results are valid once the stream has reached
 * the work.  All device pointers must be 4-byte aligned and must stay valid
 * until the work completes.
 *
 * Errors: arguments are checked on the host before anything is launched;
 * DRR_ERR_INVALID_ARG / DRR_ERR_UNSUPPORTED return without touching the
 * device.  A failed launch returns DRR_ERR_CUDA.  Faults of earlier
 * asynchronous work surface at the caller's next synchronisation, as in
 * CUDA.  drr_get_last_error() describes the last failure of this thread.
 * No C++ exception crosses the ABI.  The kernels contain no waits, so a
 * launch always terminates; a ray whose geometry is not finite (NaN/inf in
 * Rt) is treated as a miss.
 */
#ifndef DRR_H
#define DRR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DRR_API __attribute__((visibility("default")))
#else
#define DRR_API
#endif

typedef enum {
    DRR_OK = 0,
    DRR_ERR_INVALID_ARG = 1,   /* bad pointer, size, enum value or geometry */
    DRR_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. too large) */
    DRR_ERR_CUDA = 3           /* a CUDA launch or query failed */
} drr_status;

typedef enum {
    DRR_MODE_RAW = 0,          /* out = I */
    DRR_MODE_BEER_LAMBERT = 1, /* out = 1 - exp(-I), evaluated as -expm1(-I) */
    /* Front-to-back alpha compositing, the over operator (flashdrr.rendering
       API docs, VolumeRaycaster.__init__: use_beer_lambert = False), read as
       the emission-absorption sum: sample i has opacity
       a_i = 1 - exp(-density_factor * mu_i * dt) and colour mu_i, and
       out = sum_i T_i a_i mu_i with T_0 = 1, T_{i+1} = T_i (1 - a_i), summed
       from the camera side.  Its volume gradient is drr_render_alpha_adjoint
       (it is not linear in the volume); drr_render_pose_grad(_batched) take
       it too. */
    DRR_MODE_ALPHA = 2
} drr_mode;

typedef enum {
    DRR_F32 = 0,               /* float32 voxels */
    DRR_BF16 = 1               /* bfloat16 voxels (round-to-nearest-even), fp32 arithmetic */
} drr_dtype;

typedef enum {
    /* vol[k][j][i] exactly as the caller holds it (float32 or bfloat16). */
    DRR_LAYOUT_LINEAR = 0,
    /* vol[k+1][j+1][i+1] inside a one-voxel zero border: dims (nx+2, ny+2,
       nz+2).  Written by drr_prepare_volume. */
    DRR_LAYOUT_PADDED = 1,
    /* Corner-replicated: for every cell (i, j, k) in [0, nx-2] x [0, ny-2] x
       [0, nz-2] (cell index (k*(ny-1) + j)*(nx-1) + i) its 8 corner voxels
       vol[k+c][j+b][i+a] stored contiguously in the order a + 2b + 4c: 8
       elements, 16 bytes (bf16) or 32 bytes (fp32) per cell, 16-byte
       aligned.  Written by drr_prepare_volume.  One sample of the forward
       then reads its 8 voxels with one (bf16) or two (fp32) 16-byte loads
       instead of 8 scalar gathers; the price is 8x the storage. */
    DRR_LAYOUT_CORNERS = 2,
    /* xy quads: for every (i, j, k) in [0, nx-2] x [0, ny-2] x [0, nz-1]
       (quad index (k*(ny-1) + j)*(nx-1) + i) the 4 voxels vol[k][j+b][i+a]
       stored contiguously in the order a + 2b: 4 elements, 8 bytes (bf16) or
       16 bytes (fp32), 16-byte aligned.  Written by drr_prepare_volume.  A
       sample reads two quads (slices k and k+1); 4x the storage, half of the
       corner records'. */
    DRR_LAYOUT_QUADS = 3,
    /* Bricks: the cells in bricks of 8 x 8 x 8; brick (bx, by, bz), number
       (bz * nby + by) * nbx + bx with nb = ceil((n - 1) / 8) bricks per axis,
       stores the voxels vol[8bz + lz][8by + ly][8bx + lx] for lx, ly, lz in
       [0, 8] (its cells' corners: the last plane of each axis repeats the
       next brick's first), x fastest, at element (lz * 9 + ly) * 9 + lx of
       a 736-element block (zero past the 729 voxels and past the volume's
       edge).  A sample's 8 corners lie in one brick at constant offsets; the
       storage is about 1.42x the volume (96.5 MB fp32 at 256^3), so it fits
       in L2 where corner records and quads do not.  Written by
       drr_prepare_volume; 16-byte aligned. */
    DRR_LAYOUT_BRICKS = 4
} drr_layout;

/* Forward projection.
 *   vol         DEVICE, volume in `layout` and `dtype` (LINEAR: nx*ny*nz
 *               elements; other layouts: as written by drr_prepare_volume).
 *   dims        HOST int[3] {nx, ny, nz}, each in [2, 2^22 - 4].
 *   spacing     HOST float[3] voxel size (mm), > 0.
 *   origin      HOST float[3] centre of voxel 0 (mm).
 *   K           HOST float[9] intrinsics (see conventions).
 *   Rt          DEVICE float[B*12] extrinsics.
 *   B, H, W     views and detector rows / columns, >= 0 (any of them 0:
 *               nothing to do, DRR_OK); B <= 65535.
 *   n_samples   samples per ray, 1 <= n_samples <= 1048576.
 *   density_factor  finite scale of the integral.
 *   mode        DRR_MODE_RAW, DRR_MODE_BEER_LAMBERT or DRR_MODE_ALPHA.
 *   out         DEVICE float[B*H*W], overwritten.
 * Limits: the stored volume must hold fewer than 2^31 elements (PADDED:
 * with its border; CORNERS: 8 per cell; BRICKS: 736 per brick); B*H*W <
 * 2^40.  A CORNERS, QUADS or BRICKS volume must be 16-byte aligned.
 */
DRR_API drr_status drr_render(const void *vol, drr_dtype dtype, drr_layout layout,
                              const int dims[3], const float spacing[3], const float origin[3],
                              const float K[9], const float *Rt, int B, int H, int W,
                              int n_samples, float density_factor, drr_mode mode, float *out,
                              void *stream);

/* drr_render of a DRR_LAYOUT_BRICKS volume with each layer of a tile's
 * frustum staged in shared memory: the volume layout's optional staging of
 * bricks for narrow frusta.  A CTA renders a 16 x 16 pixel tile; where its
 * rays are sparse (the tile spans 8 voxels or more at the volume centre) it
 * walks the tile's pyramid one layer of 8^3-cell bricks at a time along the
 * major axis of its central ray, copying the layer's bricks (at most 16;
 * the window comes from the tile's corner rays) from global into shared
 * memory with bulk copies of the Tensor Memory Accelerator while the rays
 * sample the previous layer; denser tiles read global memory.  The result
 * is bit for bit drr_render's with DRR_LAYOUT_BRICKS (and DRR_LAYOUT_LINEAR).
 * Measured on B200 it is slower than drr_render's bricked forward on every
 * workload of this library's benchmark (one barrier per layer hides too
 * little copy latency at 2 CTAs per SM), so drr_render does not use it; it
 * is kept as the measured comparison.
 *   vol         DEVICE, DRR_LAYOUT_BRICKS as written by drr_prepare_volume,
 *               16-byte aligned.
 *   mode        DRR_MODE_RAW or DRR_MODE_BEER_LAMBERT (alpha:
 *               DRR_ERR_UNSUPPORTED).
 * Other arguments, limits and errors as drr_render. */
DRR_API drr_status drr_render_staged(const void *vol, drr_dtype dtype, const int dims[3],
                                     const float spacing[3], const float origin[3],
                                     const float K[9], const float *Rt, int B, int H, int W,
                                     int n_samples, float density_factor, drr_mode mode,
                                     float *out, void *stream);

/* Adjoint (transpose) of drr_render with respect to the volume, i.e. the
 * volume gradient of sum(grad_out * out).
 *   grad_out    DEVICE float[B*H*W], upstream gradient dL/d(out).
 *   fwd_out     DEVICE float[B*H*W], the Beer-Lambert image this gradient
 *               belongs to (required in DRR_MODE_BEER_LAMBERT, where each
 *               ray's gradient is scaled by exp(-I) = 1 - out; ignored and
 *               may be NULL in DRR_MODE_RAW).
 *   grad_vol    DEVICE float32 [nz][ny][nx] (linear layout), ACCUMULATED
 *               into with atomic adds (zero it first for a plain gradient).
 *               The order of the atomic adds is not deterministic, so results
 *               may differ between runs in the last bits.
 * Other arguments as drr_render; mode DRR_MODE_ALPHA is DRR_ERR_UNSUPPORTED
 * here (see drr_render_alpha_adjoint).  grad_vol must not overlap the images.
 */
DRR_API drr_status drr_render_adjoint(const int dims[3], const float spacing[3],
                                      const float origin[3], const float K[9], const float *Rt,
                                      int B, int H, int W, int n_samples, float density_factor,
                                      drr_mode mode, const float *grad_out, const float *fwd_out,
                                      float *grad_vol, void *stream);

/* Bytes of the workspace drr_render_adjoint_ws needs for a volume of dims
 * and B views (0 if the arguments are invalid): a header (view flags, the
 * views' camera matrices, 96 bytes per view, and a few words of
 * synchronisation, in 256-byte units) plus one 32-byte corner record per
 * cell, (nx-1)(ny-1)(nz-1) of them (about 8x the fp32 volume). */
DRR_API size_t drr_adjoint_workspace_bytes(const int dims[3], int B);

/* drr_render_adjoint with a caller-provided workspace, for speed: views
 * whose rays are much closer than a voxel (a 16-pixel tile spanning fewer
 * than 8 voxels at the volume centre) accumulate into per-cell corner
 * records with 16-byte vector atomics, which a pass then adds into
 * grad_vol.  The other views accumulate into the records of one slab of
 * cell layers at a time (a slab small enough to stay in the L2), added into
 * grad_vol after each slab; that pass is one cooperative launch, its phases
 * separated by grid-wide barriers.  A barrier wait that has not ended after
 * 20 s gives up, the pass is abandoned (grad_vol then lacks part of those
 * views' contributions) and the event is counted: drr_wait_timeouts.  The
 * pass's grid is sized to what the device reports it can hold at once; if
 * the launch is refused (fewer SMs available to the process than the
 * device has, say), the call returns DRR_ERR_CUDA.  Calls of fewer than
 * 8 * 2^20 ray-samples (B * H * W * n_samples) send their sparse views to
 * the direct path instead.  Same result as drr_render_adjoint up to fp32
 * summation order.
 *   workspace        DEVICE, 256-byte aligned, at least
 *                    drr_adjoint_workspace_bytes(dims, B) bytes; its content
 *                    on entry is ignored and on return is unspecified; must
 *                    not overlap any other buffer of the call.
 *   workspace_bytes  bytes available at workspace.
 * Calls that share one workspace must not overlap on the GPU (same stream,
 * or ordered by events).  Other arguments as drr_render_adjoint. */
DRR_API drr_status drr_render_adjoint_ws(const int dims[3], const float spacing[3],
                                         const float origin[3], const float K[9],
                                         const float *Rt, int B, int H, int W, int n_samples,
                                         float density_factor, drr_mode mode,
                                         const float *grad_out, const float *fwd_out,
                                         float *grad_vol, void *workspace,
                                         size_t workspace_bytes, void *stream);

/* Grid-barrier waits of the slab pass (drr_render_adjoint_ws and the calls
 * built on it) that gave up on the current device since the last call; the
 * count is cleared.  0 in normal operation: every CTA of the cooperative
 * launch is resident, so a wait ends when the slowest CTA arrives.  Reads
 * device memory synchronously (call it once the work has completed).
 * Returns DRR_OK, DRR_ERR_INVALID_ARG for a NULL count, or DRR_ERR_CUDA. */
DRR_API drr_status drr_wait_timeouts(unsigned long long *count);

/* Size of the scratch built into the library for drr_render_adjoint_noalloc. */
#define DRR_NOALLOC_SCRATCH_BYTES (32u << 20)

/* drr_render_adjoint_ws without a caller-provided workspace, for callers
 * that may not allocate device memory: code running under a memory manager
 * that owns all of the device's memory (a framework's caching allocator, a
 * server with fixed per-model budgets), or a real-time loop in which an
 * allocation, which can synchronise the device, is not allowed.  The pages
 * this library follows have no counterpart of this call; it exists only for
 * such callers.
 *   - The workspace is a scratch array built into the library's device
 *     image, DRR_NOALLOC_SCRATCH_BYTES (32 MiB) in size.  Every GPU that
 *     loads the library holds it until the process exits.
 *   - Volumes and view counts whose workspace
 *     (drr_adjoint_workspace_bytes(dims, B)) exceeds that size are rejected
 *     with DRR_ERR_UNSUPPORTED before anything runs (about 100^3 voxels at
 *     most); use drr_render_adjoint_ws for larger ones.
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library
 *     call.  The first call on a device looks up the scratch's device
 *     address (once per device, with that device current); make that first
 *     call before any stream capture.  The address is cached for the life
 *     of the process: do not call cudaDeviceReset between calls (the cached
 *     address would be stale).  The scratch used is the one of the device
 *     current on the calling thread, so that device must be the one that
 *     owns `stream` and the buffers.
 *   - Argument checks are those of drr_render_adjoint_ws; a rejected call
 *     touches nothing on the device.
 *   - All calls share the one scratch array, which keeps the last call's
 *     contents; each call re-initialises what it reads.  Calls that overlap
 *     on the GPU (different streams without ordering, or several host
 *     threads) race on it: serialise them.
 * Arguments and result as drr_render_adjoint. */
DRR_API drr_status drr_render_adjoint_noalloc(const int dims[3], const float spacing[3],
                                              const float origin[3], const float K[9],
                                              const float *Rt, int B, int H, int W,
                                              int n_samples, float density_factor,
                                              drr_mode mode, const float *grad_out,
                                              const float *fwd_out, float *grad_vol,
                                              void *stream);

/* Pose gradient: dL/d[R|t] of L = sum(grad_out * out), per view, for the
 * registration use of a differentiable renderer (flashdrr.rendering API
 * docs, VolumeRaycaster: rendering is differentiable with respect to the
 * view matrices; FlashDRR page, 2D/3D registration).  The 12 entries of
 * each view's world-to-camera matrix are taken as free variables of the ray
 * as written: direction R^T K^-1 (u, v, 1) normalised, centre -R^T t.
 * Along rotations (dR = R [w]x) this equals the derivative of any rotation
 * parameterisation; off the rotation group it is the derivative of these
 * formulas (R^T, not R^-1).  The chain rule runs through the clip (each end
 * moves with the box plane it lies on; an entry point at the camera, when
 * the camera is inside the box, does not move), the sample positions, the
 * gradient of the trilinear interpolant inside each sample's cell and dt.
 * In DRR_MODE_ALPHA each sample's gradient is weighted by dC/dmu_i (see
 * drr_render_alpha_adjoint) and dt enters through the opacities as well:
 * dC/ds = sum_i T_i mu_i^2 (1 - a_i) - mu_i (C - C_i), s = density_factor dt.
 *   vol, dtype, layout  the forward's volume (any layout).
 *   grad_out    DEVICE float[B*H*W], upstream gradient dL/d(out).
 *   fwd_out     DEVICE float[B*H*W], the forward's image: required in
 *               DRR_MODE_BEER_LAMBERT (each ray's term is scaled by
 *               exp(-I) = 1 - out) and in DRR_MODE_ALPHA (the composite C
 *               of each ray); may be NULL in DRR_MODE_RAW.
 *   grad_Rt     DEVICE float[B*12], row-major like Rt, ACCUMULATED into (zero
 *               it first for a plain gradient); must not overlap Rt or the
 *               images.  Per-ray terms are formed in fp64 and summed per CTA
 *               in fp64, then added with fp32 atomics (order not
 *               deterministic: the last bits may differ between runs).
 * Other arguments as drr_render. */
DRR_API drr_status drr_render_pose_grad(const void *vol, drr_dtype dtype, drr_layout layout,
                                        const int dims[3], const float spacing[3],
                                        const float origin[3], const float K[9],
                                        const float *Rt, int B, int H, int W, int n_samples,
                                        float density_factor, drr_mode mode,
                                        const float *grad_out, const float *fwd_out,
                                        float *grad_Rt, void *stream);

/* Pose gradient of drr_render_batched (any mode): grad_Rt, DEVICE
 * float[n_views * 12], ACCUMULATED into; each image adds its terms to the
 * pose it was rendered from (with n_views == 1, every volume's image adds to
 * pose 0).  vols, Rt, grad_out and fwd_out as drr_render_batched and
 * drr_render_adjoint_batched; other arguments as drr_render_pose_grad. */
DRR_API drr_status drr_render_pose_grad_batched(const void *vols, drr_dtype dtype,
                                                drr_layout layout, const int dims[3],
                                                const float spacing[3], const float origin[3],
                                                const float K[9], const float *Rt, int n_vols,
                                                int channels, int n_views, int H, int W,
                                                int n_samples, float density_factor,
                                                drr_mode mode, const float *grad_out,
                                                const float *fwd_out, float *grad_Rt,
                                                void *stream);

/* Volume gradient of a DRR_MODE_ALPHA image: grad_vol += d(sum grad_out *
 * out)/d vol.  With C_i the composite up to and including sample i and C the
 * ray's image value, dC/dmu_i = T_i (s (1 - a_i) mu_i + a_i) - s (C - C_i),
 * s = density_factor * dt; each sample's value is scattered with its
 * trilinear weights.  One pass per ray, front to back.
 *   vol, dtype, layout  the forward's volume: DRR_LAYOUT_LINEAR,
 *               DRR_LAYOUT_CORNERS, DRR_LAYOUT_QUADS or DRR_LAYOUT_BRICKS
 *               (DRR_LAYOUT_PADDED: DRR_ERR_UNSUPPORTED).
 *   grad_out    DEVICE float[B*H*W], upstream gradient dL/d(out).
 *   fwd_out     DEVICE float[B*H*W], the alpha image of this volume and these
 *               poses (drr_render with DRR_MODE_ALPHA), required.
 *   grad_vol    DEVICE float32 [nz][ny][nx], ACCUMULATED into (atomic adds,
 *               order not deterministic); must not overlap the other buffers.
 * Other arguments as drr_render. */
DRR_API drr_status drr_render_alpha_adjoint(const void *vol, drr_dtype dtype, drr_layout layout,
                                            const int dims[3], const float spacing[3],
                                            const float origin[3], const float K[9],
                                            const float *Rt, int B, int H, int W, int n_samples,
                                            float density_factor, const float *grad_out,
                                            const float *fwd_out, float *grad_vol, void *stream);

/* drr_render_alpha_adjoint with a caller-provided workspace, for speed:
 * views whose rays are much closer than a voxel (the test of
 * drr_render_adjoint_ws) accumulate into per-cell corner records, which a
 * final pass adds into grad_vol; other views scatter directly.  Same result
 * up to fp32 summation order.
 *   workspace        DEVICE, 256-byte aligned, at least
 *                    drr_adjoint_workspace_bytes(dims, B) bytes; content on
 *                    entry ignored, on return unspecified; must not overlap
 *                    any other buffer of the call.
 *   workspace_bytes  bytes available at workspace.
 * Calls that share one workspace must not overlap on the GPU.  Other
 * arguments as drr_render_alpha_adjoint. */
DRR_API drr_status drr_render_alpha_adjoint_ws(const void *vol, drr_dtype dtype, drr_layout layout,
                                               const int dims[3], const float spacing[3],
                                               const float origin[3], const float K[9],
                                               const float *Rt, int B, int H, int W,
                                               int n_samples, float density_factor,
                                               const float *grad_out, const float *fwd_out,
                                               float *grad_vol, void *workspace,
                                               size_t workspace_bytes, void *stream);

/* Volume gradient of a batched DRR_MODE_ALPHA render (drr_render_batched):
 * grad_vols, DEVICE float32 [n_vols * channels][nz][ny][nx] (linear),
 * ACCUMULATED into; each image's gradient goes to the volume-channel it was
 * rendered from.  workspace: NULL (every image on the direct path) or at
 * least drr_adjoint_batched_workspace_bytes(dims, n_vols, channels, n_views)
 * bytes, 256-byte aligned (dense images accumulate into the corner records of
 * their volume-channel).  vols, Rt, grad_out and fwd_out (the batched alpha
 * image, required) as drr_render_batched; other arguments as
 * drr_render_alpha_adjoint_ws. */
DRR_API drr_status drr_render_alpha_adjoint_batched(const void *vols, drr_dtype dtype,
                                                    drr_layout layout, const int dims[3],
                                                    const float spacing[3], const float origin[3],
                                                    const float K[9], const float *Rt,
                                                    int n_vols, int channels, int n_views, int H,
                                                    int W, int n_samples, float density_factor,
                                                    const float *grad_out, const float *fwd_out,
                                                    float *grad_vols, void *workspace,
                                                    size_t workspace_bytes, void *stream);

/* Gaussian-Poisson surrogate of shot noise (flashdrr.rendering API docs,
 * VolumeRaycaster.apply_poisson) on a Beer-Lambert image: with transmission
 * T = 1 - image, T' = clamp(T + sqrt(T / i0) z, 0, 1) and out = 1 - T'.
 *   image   DEVICE float[n], a Beer-Lambert image (values in [0, 1]).
 *   z       DEVICE float[n], standard normal draws (the caller's generator).
 *   i0      mean photon count at the source, finite and > 0.
 *   out     DEVICE float[n]; may be image itself (in place), must not
 *           overlap z or only part of image.
 * n == 0 is a no-op. */
DRR_API drr_status drr_poisson_noise(const float *image, const float *z, float i0, float *out,
                                     int64_t n, void *stream);

/* Its derivative: grad_image = grad_out * (1 + z / (2 sqrt(T i0))) where the
 * clamp is inactive (0 < T + sqrt(T / i0) z < 1, T > 0), else 0.
 *   grad_image  DEVICE float[n], overwritten; may be grad_out itself, must not
 *               overlap image or z.
 * Other arguments as drr_poisson_noise. */
DRR_API drr_status drr_poisson_noise_backward(const float *image, const float *z, float i0,
                                              const float *grad_out, float *grad_image,
                                              int64_t n, void *stream);

/* The cell-constant (Siddon) projector (diffct page, Features: project()
 * and backproject() form an exact adjoint pair for the cell-constant Siddon
 * model): a second discretisation of the same line integral.  Voxel
 * (i, j, k) is the cube of side one voxel centred on (i, j, k) in IJK, with
 * the constant value vol[k][j][i]; a ray's image is density_factor times the
 * exact integral of that piecewise-constant function along the ray (the sum
 * over the cells it crosses of chord length in mm times value), clipped to
 * the cells' box [-1/2, n - 1/2] per axis (t0 = max(t_near, 0)), written raw
 * or as 1 - exp(-I).  No samples: n_samples does not apply.
 *   vol     DEVICE, DRR_LAYOUT_LINEAR only, fp32 or bf16.
 *   mode    DRR_MODE_RAW or DRR_MODE_BEER_LAMBERT (DRR_MODE_ALPHA:
 *           DRR_ERR_UNSUPPORTED).
 * Other arguments as drr_render. */
DRR_API drr_status drr_render_siddon(const void *vol, drr_dtype dtype, const int dims[3],
                                     const float spacing[3], const float origin[3],
                                     const float K[9], const float *Rt, int B, int H, int W,
                                     float density_factor, drr_mode mode, float *out,
                                     void *stream);

/* Its exact adjoint (the matched backprojection): grad_vol += each ray's
 * grad_out * density_factor (times exp(-I) = 1 - fwd_out in Beer-Lambert)
 * times its chord length in every cell it crosses; fp32 atomic adds, order
 * not deterministic.  Arguments as drr_render_adjoint without n_samples. */
DRR_API drr_status drr_render_siddon_adjoint(const int dims[3], const float spacing[3],
                                             const float origin[3], const float K[9],
                                             const float *Rt, int B, int H, int W,
                                             float density_factor, drr_mode mode,
                                             const float *grad_out, const float *fwd_out,
                                             float *grad_vol, void *stream);

/* Batches of volumes, channels and views (flashdrr.rendering API docs,
 * VolumeRaycaster.forward: vol of shape (B, C, D, H, W) and view matrices of
 * shape (N, 4, 4) with N = B * views_per_vol, N == 1 broadcast to B; output
 * (N, C, H, W)).
 *   vols      DEVICE: n_vols * channels volumes of one geometry, each in
 *             `layout` and `dtype` (drr_prepared_bytes(dims, dtype, layout)
 *             bytes each), back to back: volume v, channel ch at slot
 *             v * channels + ch.
 *   Rt        DEVICE float[n_views * 12]: n_views == 1 renders that pose of
 *             every volume (n_out = n_vols); otherwise n_views must be a
 *             multiple of n_vols, and views v * views_per_vol ...
 *             (v + 1) * views_per_vol - 1 see volume v (n_out = n_views,
 *             views_per_vol = n_views / n_vols).
 *   out       DEVICE float[n_out * channels * H * W], image (n, ch) at
 *             n * channels + ch.
 * n_out * channels <= 65535.  Other arguments and modes as drr_render. */
DRR_API drr_status drr_render_batched(const void *vols, drr_dtype dtype, drr_layout layout,
                                      const int dims[3], const float spacing[3],
                                      const float origin[3], const float K[9], const float *Rt,
                                      int n_vols, int channels, int n_views, int H, int W,
                                      int n_samples, float density_factor, drr_mode mode,
                                      float *out, void *stream);

/* Adjoint of drr_render_batched (RAW or Beer-Lambert): grad_vols, DEVICE
 * float32 [n_vols * channels][nz][ny][nx] (linear), ACCUMULATED into; each
 * image's gradient goes to the volume-channel it was rendered from.  Uses
 * the direct scatter path (no workspace; see drr_render_adjoint_batched_ws).
 * Other arguments as drr_render_adjoint and drr_render_batched. */
DRR_API drr_status drr_render_adjoint_batched(const int dims[3], const float spacing[3],
                                              const float origin[3], const float K[9],
                                              const float *Rt, int n_vols, int channels,
                                              int n_views, int H, int W, int n_samples,
                                              float density_factor, drr_mode mode,
                                              const float *grad_out, const float *fwd_out,
                                              float *grad_vols, void *stream);

/* Bytes of the workspace drr_render_adjoint_batched_ws needs (0 if the
 * arguments are invalid): a 256-byte aligned header of one int per output
 * image plus one, then the corner records (32 bytes per cell,
 * (nx-1)(ny-1)(nz-1) cells) of each of the n_vols * channels
 * volume-channels. */
DRR_API size_t drr_adjoint_batched_workspace_bytes(const int dims[3], int n_vols, int channels,
                                                   int n_views);

/* drr_render_adjoint_batched with a caller-provided workspace, for speed:
 * images whose rays are much closer than a voxel (the test of
 * drr_render_adjoint_ws) accumulate into the corner records of their
 * volume-channel, which a final pass adds into grad_vols; other images
 * scatter directly.  Same result up to fp32 summation order.
 *   workspace        DEVICE, 256-byte aligned, at least
 *                    drr_adjoint_batched_workspace_bytes(dims, n_vols,
 *                    channels, n_views) bytes; content on entry ignored, on
 *                    return unspecified; must not overlap any other buffer
 *                    of the call.
 *   workspace_bytes  bytes available at workspace.
 * Calls that share one workspace must not overlap on the GPU.  Other
 * arguments as drr_render_adjoint_batched. */
DRR_API drr_status drr_render_adjoint_batched_ws(const int dims[3], const float spacing[3],
                                                 const float origin[3], const float K[9],
                                                 const float *Rt, int n_vols, int channels,
                                                 int n_views, int H, int W, int n_samples,
                                                 float density_factor, drr_mode mode,
                                                 const float *grad_out, const float *fwd_out,
                                                 float *grad_vols, void *workspace,
                                                 size_t workspace_bytes, void *stream);

/* Bytes that drr_prepare_volume writes for this volume, dtype and layout
 * (0 if the arguments are invalid or the volume is too large). */
DRR_API size_t drr_prepared_bytes(const int dims[3], drr_dtype dtype, drr_layout layout);

/* Re-lay-out (and optionally convert) a volume for drr_render.
 *   src         DEVICE float32 [nz][ny][nx].
 *   dst         DEVICE, at least drr_prepared_bytes(dims, dtype, layout)
 *               bytes (dst_bytes says how many are available); must not
 *               overlap src; 16-byte aligned for DRR_LAYOUT_CORNERS, _QUADS
 *               and _BRICKS.  Every
 *               byte of the prepared volume is written.
 * bf16 conversion rounds to nearest even.  Done once per volume (or once per
 * update of the volume), not per render. */
DRR_API drr_status drr_prepare_volume(const float *src, const int dims[3], drr_dtype dtype,
                                      drr_layout layout, void *dst, size_t dst_bytes,
                                      void *stream);

/* Human-readable description of the last failure on this thread ("" if
 * none).  The string stays valid until the next call on this thread. */
DRR_API const char *drr_get_last_error(void);

/* ABI version of this header: 1. */
DRR_API int drr_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DRR_H */

// drr_api.cu -- the extern "C" entry points of libdrr.so (include/drr.h).
//
// Host side only: validate every argument before touching the device,
// precompute K^-1 in double, fill the kernel parameter block and launch on
// the caller's stream.  No allocation, no synchronisation, no state kept
// between calls (the last-error string is per thread).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>

#include "../../include/drr.h"
#include "../../include/drr_debug.h"
#include "drr_internal.cuh"

static_assert(DRR_NOALLOC_SCRATCH_BYTES == drr::kNoAllocScratchBytes,
              "the header's scratch size must be the library's");

namespace {

thread_local char g_last_error[512] = "";

drr_status fail(drr_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

drr_status ok() {
    g_last_error[0] = '\0';
    return DRR_OK;
}

drr_status cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return ok();
    return fail(DRR_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int kMaxSamples = 1 << 20;
constexpr int kMaxViews = 65535;
constexpr int kMaxRows = 65535 * drr::kTileH;
constexpr int64_t kMaxElements = (int64_t(1) << 31) - 1;
constexpr int kMaxDim = (1 << 22) - 4;   // keeps padded coordinates inside the exact floor range

bool known_layout(int layout) {
    return layout == DRR_LAYOUT_LINEAR || layout == DRR_LAYOUT_PADDED ||
           layout == DRR_LAYOUT_CORNERS || layout == DRR_LAYOUT_QUADS ||
           layout == DRR_LAYOUT_BRICKS;
}

int64_t stored_elements(const int dims[3], int layout) {
    if (layout == DRR_LAYOUT_CORNERS)
        return (int64_t)(dims[0] - 1) * (dims[1] - 1) * (dims[2] - 1) * 8;
    if (layout == DRR_LAYOUT_QUADS) return (int64_t)(dims[0] - 1) * (dims[1] - 1) * dims[2] * 4;
    if (layout == DRR_LAYOUT_BRICKS)
        return (int64_t)drr::brick_count(dims[0]) * drr::brick_count(dims[1]) *
               drr::brick_count(dims[2]) * drr::kBrickStride;
    const int pad = layout == DRR_LAYOUT_PADDED ? 2 : 0;
    return (int64_t)(dims[0] + pad) * (dims[1] + pad) * (dims[2] + pad);
}

size_t layout_alignment(int layout, int dtype) {
    if (layout == DRR_LAYOUT_CORNERS || layout == DRR_LAYOUT_QUADS || layout == DRR_LAYOUT_BRICKS)
        return 16;
    return dtype == DRR_F32 ? 4 : 2;
}

drr_status check_volume(const int dims[3], const float spacing[3], const float origin[3]) {
    if (!dims || !spacing || !origin) return fail(DRR_ERR_INVALID_ARG, "dims, spacing and origin must be non-NULL");
    for (int a = 0; a < 3; ++a) {
        if (dims[a] < 2 || dims[a] > kMaxDim)
            return fail(DRR_ERR_INVALID_ARG, "dims[%d] = %d must be in [2, %d]", a, dims[a], kMaxDim);
        if (!(spacing[a] > 0.0f) || !std::isfinite(spacing[a]))
            return fail(DRR_ERR_INVALID_ARG, "spacing[%d] must be finite and > 0", a);
        if (!std::isfinite(origin[a])) return fail(DRR_ERR_INVALID_ARG, "origin[%d] must be finite", a);
    }
    return DRR_OK;
}

drr_status check_rays(const float K[9], const float* Rt, int B, int H, int W, int n_samples,
                      float density_factor, int mode, bool alpha_ok = false) {
    if (!K) return fail(DRR_ERR_INVALID_ARG, "K must be a non-NULL host array of 9 floats");
    for (int m = 0; m < 9; ++m)
        if (!std::isfinite(K[m])) return fail(DRR_ERR_INVALID_ARG, "K[%d] is not finite", m);
    if (K[3] != 0.0f || K[6] != 0.0f || K[7] != 0.0f)
        return fail(DRR_ERR_INVALID_ARG, "K must be upper triangular (K[3] = K[6] = K[7] = 0)");
    if (K[0] == 0.0f || K[4] == 0.0f || K[8] == 0.0f)
        return fail(DRR_ERR_INVALID_ARG, "K must be invertible (K[0], K[4], K[8] non-zero)");
    if (B < 0 || H < 0 || W < 0) return fail(DRR_ERR_INVALID_ARG, "B, H, W must be >= 0");
    if (B > kMaxViews) return fail(DRR_ERR_UNSUPPORTED, "B = %d exceeds %d views per call", B, kMaxViews);
    if (H > kMaxRows) return fail(DRR_ERR_UNSUPPORTED, "H = %d exceeds %d rows", H, kMaxRows);
    if ((int64_t)B * H * W >= (int64_t(1) << 40)) return fail(DRR_ERR_UNSUPPORTED, "B*H*W too large");
    if (n_samples < 1 || n_samples > kMaxSamples)
        return fail(DRR_ERR_INVALID_ARG, "n_samples = %d must be in [1, %d]", n_samples, kMaxSamples);
    if (!std::isfinite(density_factor)) return fail(DRR_ERR_INVALID_ARG, "density_factor must be finite");
    if (mode == DRR_MODE_ALPHA && !alpha_ok)
        return fail(DRR_ERR_UNSUPPORTED,
                    "DRR_MODE_ALPHA is not linear in the volume: its gradient needs the volume "
                    "(drr_render_alpha_adjoint)");
    if (mode != DRR_MODE_RAW && mode != DRR_MODE_BEER_LAMBERT && mode != DRR_MODE_ALPHA)
        return fail(DRR_ERR_INVALID_ARG, "unknown mode %d", mode);
    if ((int64_t)B * H * W > 0 && (!Rt || !aligned(Rt, 4)))
        return fail(DRR_ERR_INVALID_ARG, "Rt must be a non-NULL, 4-byte aligned device pointer");
    return DRR_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

// The batch rule of VolumeRaycaster.forward: n_views view matrices for
// n_vols volumes of `channels` channels; n_views == 1 is broadcast to every
// volume, else n_views must be a multiple of n_vols (views_per_vol of them
// per volume, consecutive).  Output images: n_out x channels.
drr_status batch_shape(int n_vols, int channels, int n_views, int* n_out, int* per_vol,
                       int* broadcast) {
    if (n_vols < 0 || channels < 0 || n_views < 0)
        return fail(DRR_ERR_INVALID_ARG, "n_vols, channels and n_views must be >= 0");
    if (n_vols == 0 || channels == 0 || n_views == 0) {
        *n_out = 0;
        *per_vol = 1;
        *broadcast = 0;
        return DRR_OK;
    }
    if (n_views == 1 && n_vols > 1) {
        *n_out = n_vols;
        *per_vol = 1;
        *broadcast = 1;
    } else if (n_views % n_vols == 0) {
        *n_out = n_views;
        *per_vol = n_views / n_vols;
        *broadcast = 0;
    } else {
        return fail(DRR_ERR_INVALID_ARG,
                    "n_views = %d must be 1 or a multiple of n_vols = %d", n_views, n_vols);
    }
    if ((int64_t)*n_out * channels > kMaxViews)
        return fail(DRR_ERR_UNSUPPORTED, "%lld images (views x channels) exceed %d per call",
                    (long long)*n_out * channels, kMaxViews);
    return DRR_OK;
}

// The implementations, over batches of volumes x channels x views; each
// single-volume entry point is the case n_vols = channels = 1, n_views = B.

drr_status render_batched(const void* vols, drr_dtype dtype, drr_layout layout, const int dims[3],
                          const float spacing[3], const float origin[3], const float K[9],
                          const float* Rt, int n_vols, int channels, int n_views, int H, int W,
                          int n_samples, float density_factor, drr_mode mode, float* out,
                          void* stream) {
    int n_out = 0, per_vol = 1, bcast = 0;
    drr_status st = batch_shape(n_vols, channels, n_views, &n_out, &per_vol, &bcast);
    if (st != DRR_OK) return st;
    st = check_volume(dims, spacing, origin);
    if (st != DRR_OK) return st;
    const int images = n_out * channels;
    st = check_rays(K, Rt, images, H, W, n_samples, density_factor, mode, true);
    if (st != DRR_OK) return st;
    if (dtype != DRR_F32 && dtype != DRR_BF16) return fail(DRR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (!known_layout(layout)) return fail(DRR_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (stored_elements(dims, layout) > kMaxElements)
        return fail(DRR_ERR_UNSUPPORTED, "volume too large (max 2^31 - 1 stored elements)");
    if ((int64_t)images * H * W == 0) return ok();
    if (!vols || !aligned(vols, layout_alignment(layout, dtype)))
        return fail(DRR_ERR_INVALID_ARG, "vols must be a non-NULL device pointer aligned to %zu bytes",
                    layout_alignment(layout, dtype));
    if (!out || !aligned(out, 4)) return fail(DRR_ERR_INVALID_ARG, "out must be a non-NULL, 4-byte aligned device pointer");
    drr::Geom g;
    drr::fill_geom(g, dims, spacing, origin, K, images, H, W, n_samples, density_factor, layout);
    g.C = channels;
    g.views_per_vol = per_vol;
    g.broadcast = bcast;
    g.vstride = stored_elements(dims, layout);
    return cuda_status(drr::launch_forward(vols, dtype, layout, g, Rt, mode, out,
                                           static_cast<cudaStream_t>(stream)),
                       "drr_render launch");
}

// Where the adjoint's workspace comes from: none (every view on the direct
// path), the caller's buffer, or the library's built-in scratch (the
// allocation-free entry point).
enum class Workspace { kNone, kCaller, kBuiltin };

drr_status render_adjoint_batched(const int dims[3], const float spacing[3], const float origin[3],
                                  const float K[9], const float* Rt, int n_vols, int channels,
                                  int n_views, int H, int W, int n_samples, float density_factor,
                                  drr_mode mode, const float* grad_out, const float* fwd_out,
                                  float* grad_vols, Workspace ws_kind, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    int n_out = 0, per_vol = 1, bcast = 0;
    drr_status st = batch_shape(n_vols, channels, n_views, &n_out, &per_vol, &bcast);
    if (st != DRR_OK) return st;
    st = check_volume(dims, spacing, origin);
    if (st != DRR_OK) return st;
    const int images = n_out * channels;
    st = check_rays(K, Rt, images, H, W, n_samples, density_factor, mode);
    if (st != DRR_OK) return st;
    if (stored_elements(dims, DRR_LAYOUT_LINEAR) > kMaxElements)
        return fail(DRR_ERR_UNSUPPORTED, "volume too large (max 2^31 - 1 elements)");
    const int64_t npix = (int64_t)images * H * W;
    if (npix == 0) return ok();
    if (!grad_out || !aligned(grad_out, 4))
        return fail(DRR_ERR_INVALID_ARG, "grad_out must be a non-NULL, 4-byte aligned device pointer");
    if (mode == DRR_MODE_BEER_LAMBERT && (!fwd_out || !aligned(fwd_out, 4)))
        return fail(DRR_ERR_INVALID_ARG, "fwd_out is required in Beer-Lambert mode");
    if (!grad_vols || !aligned(grad_vols, 4))
        return fail(DRR_ERR_INVALID_ARG, "grad_vols must be a non-NULL, 4-byte aligned device pointer");
    const int64_t nvox = (int64_t)dims[0] * dims[1] * dims[2];
    const size_t vbytes = (size_t)nvox * n_vols * channels * 4, ibytes = (size_t)npix * 4;
    if (overlaps(grad_vols, vbytes, grad_out, ibytes) ||
        (mode == DRR_MODE_BEER_LAMBERT && overlaps(grad_vols, vbytes, fwd_out, ibytes)))
        return fail(DRR_ERR_INVALID_ARG, "grad_vols overlaps an image buffer");
    const size_t need =
        drr::adjoint_workspace_bytes(dims[0], dims[1], dims[2], images, n_vols * channels);
    if (ws_kind == Workspace::kBuiltin) {
        // checked before the scratch's address is looked up, so that a call
        // rejected here touches nothing on the device
        if (need > drr::kNoAllocScratchBytes)
            return fail(DRR_ERR_UNSUPPORTED,
                        "this volume and view count need %zu bytes of scratch; the built-in "
                        "scratch holds %zu (use drr_render_adjoint_ws with a workspace of your own)",
                        need, drr::kNoAllocScratchBytes);
        const cudaError_t e = drr::noalloc_scratch(&workspace);
        if (e != cudaSuccess) return cuda_status(e, "drr_render_adjoint_noalloc scratch lookup");
    } else if (ws_kind == Workspace::kCaller) {
        if (!workspace || !aligned(workspace, 256))
            return fail(DRR_ERR_INVALID_ARG, "workspace must be a non-NULL, 256-byte aligned device pointer");
        if (workspace_bytes < need)
            return fail(DRR_ERR_INVALID_ARG, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
        if (overlaps(workspace, need, grad_vols, vbytes) || overlaps(workspace, need, grad_out, ibytes) ||
            (mode == DRR_MODE_BEER_LAMBERT && overlaps(workspace, need, fwd_out, ibytes)) ||
            overlaps(workspace, need, Rt, (size_t)n_views * 12 * sizeof(float)))
            return fail(DRR_ERR_INVALID_ARG, "workspace overlaps another buffer");
    }
    drr::Geom g;
    drr::fill_geom(g, dims, spacing, origin, K, images, H, W, n_samples, density_factor,
                   DRR_LAYOUT_LINEAR);
    g.C = channels;
    g.views_per_vol = per_vol;
    g.broadcast = bcast;
    g.vstride = nvox;
    return cuda_status(drr::launch_adjoint(g, Rt, mode, grad_out, fwd_out, grad_vols,
                                           ws_kind == Workspace::kNone ? nullptr : workspace,
                                           static_cast<cudaStream_t>(stream)),
                       "drr_render_adjoint_batched launch");
}

drr_status pose_grad_batched(const void* vols, drr_dtype dtype, drr_layout layout,
                             const int dims[3], const float spacing[3], const float origin[3],
                             const float K[9], const float* Rt, int n_vols, int channels,
                             int n_views, int H, int W, int n_samples, float density_factor,
                             drr_mode mode, const float* grad_out, const float* fwd_out,
                             float* grad_Rt, void* stream) {
    int n_out = 0, per_vol = 1, bcast = 0;
    drr_status st = batch_shape(n_vols, channels, n_views, &n_out, &per_vol, &bcast);
    if (st != DRR_OK) return st;
    st = check_volume(dims, spacing, origin);
    if (st != DRR_OK) return st;
    const int images = n_out * channels;
    st = check_rays(K, Rt, images, H, W, n_samples, density_factor, mode, true);
    if (st != DRR_OK) return st;
    if (dtype != DRR_F32 && dtype != DRR_BF16) return fail(DRR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (!known_layout(layout)) return fail(DRR_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (stored_elements(dims, layout) > kMaxElements)
        return fail(DRR_ERR_UNSUPPORTED, "volume too large (max 2^31 - 1 stored elements)");
    const int64_t npix = (int64_t)images * H * W;
    if (npix == 0) return ok();
    if (!vols || !aligned(vols, layout_alignment(layout, dtype)))
        return fail(DRR_ERR_INVALID_ARG, "vols must be a non-NULL device pointer aligned to %zu bytes",
                    layout_alignment(layout, dtype));
    if (!grad_out || !aligned(grad_out, 4))
        return fail(DRR_ERR_INVALID_ARG, "grad_out must be a non-NULL, 4-byte aligned device pointer");
    if (mode != DRR_MODE_RAW && (!fwd_out || !aligned(fwd_out, 4)))
        return fail(DRR_ERR_INVALID_ARG, "fwd_out is required in Beer-Lambert and alpha mode");
    if (!grad_Rt || !aligned(grad_Rt, 4))
        return fail(DRR_ERR_INVALID_ARG, "grad_Rt must be a non-NULL, 4-byte aligned device pointer");
    const size_t gbytes = (size_t)n_views * 12 * sizeof(float), ibytes = (size_t)npix * 4;
    if (overlaps(grad_Rt, gbytes, grad_out, ibytes) || overlaps(grad_Rt, gbytes, Rt, gbytes) ||
        (mode != DRR_MODE_RAW && overlaps(grad_Rt, gbytes, fwd_out, ibytes)))
        return fail(DRR_ERR_INVALID_ARG, "grad_Rt overlaps another buffer");
    drr::Geom g;
    drr::fill_geom(g, dims, spacing, origin, K, images, H, W, n_samples, density_factor, layout);
    g.C = channels;
    g.views_per_vol = per_vol;
    g.broadcast = bcast;
    g.vstride = stored_elements(dims, layout);
    return cuda_status(drr::launch_pose_grad(vols, dtype, layout, g, Rt, mode, grad_out, fwd_out,
                                             grad_Rt, static_cast<cudaStream_t>(stream)),
                       "drr_render_pose_grad launch");
}

drr_status render_alpha_adjoint(const void* vol, drr_dtype dtype, drr_layout layout,
                                const int dims[3], const float spacing[3], const float origin[3],
                                const float K[9], const float* Rt, int n_vols, int channels,
                                int n_views, int H, int W, int n_samples, float density_factor,
                                const float* grad_out, const float* fwd_out, float* grad_vol,
                                bool with_ws, void* workspace, size_t workspace_bytes,
                                void* stream) {
    int n_out = 0, per_vol = 1, bcast = 0;
    drr_status st = batch_shape(n_vols, channels, n_views, &n_out, &per_vol, &bcast);
    if (st != DRR_OK) return st;
    st = check_volume(dims, spacing, origin);
    if (st != DRR_OK) return st;
    const int images = n_out * channels;
    st = check_rays(K, Rt, images, H, W, n_samples, density_factor, DRR_MODE_ALPHA, true);
    if (st != DRR_OK) return st;
    if (dtype != DRR_F32 && dtype != DRR_BF16) return fail(DRR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (!known_layout(layout)) return fail(DRR_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (layout == DRR_LAYOUT_PADDED)
        return fail(DRR_ERR_UNSUPPORTED,
                    "the alpha adjoint reads DRR_LAYOUT_LINEAR, _CORNERS, _QUADS or _BRICKS volumes");
    if (stored_elements(dims, layout) > kMaxElements)
        return fail(DRR_ERR_UNSUPPORTED, "volume too large (max 2^31 - 1 stored elements)");
    const int64_t npix = (int64_t)images * H * W;
    if (npix == 0) return ok();
    if (!vol || !aligned(vol, layout_alignment(layout, dtype)))
        return fail(DRR_ERR_INVALID_ARG, "vol must be a non-NULL device pointer aligned to %zu bytes",
                    layout_alignment(layout, dtype));
    if (!grad_out || !aligned(grad_out, 4))
        return fail(DRR_ERR_INVALID_ARG, "grad_out must be a non-NULL, 4-byte aligned device pointer");
    if (!fwd_out || !aligned(fwd_out, 4))
        return fail(DRR_ERR_INVALID_ARG, "fwd_out (the alpha image) is required");
    if (!grad_vol || !aligned(grad_vol, 4))
        return fail(DRR_ERR_INVALID_ARG, "grad_vol must be a non-NULL, 4-byte aligned device pointer");
    const int slots = n_vols * channels;
    const size_t vbytes = (size_t)dims[0] * dims[1] * dims[2] * 4 * slots, ibytes = (size_t)npix * 4;
    const size_t sbytes = (size_t)stored_elements(dims, layout) * (dtype == DRR_F32 ? 4 : 2) * slots;
    if (overlaps(grad_vol, vbytes, grad_out, ibytes) || overlaps(grad_vol, vbytes, fwd_out, ibytes) ||
        overlaps(grad_vol, vbytes, vol, sbytes))
        return fail(DRR_ERR_INVALID_ARG, "grad_vol overlaps another buffer");
    if (with_ws) {
        const size_t need = drr::adjoint_workspace_bytes(dims[0], dims[1], dims[2], images, slots);
        if (!workspace || !aligned(workspace, 256))
            return fail(DRR_ERR_INVALID_ARG, "workspace must be a non-NULL, 256-byte aligned device pointer");
        if (workspace_bytes < need)
            return fail(DRR_ERR_INVALID_ARG, "workspace holds %zu bytes, %zu needed", workspace_bytes, need);
        if (overlaps(workspace, need, grad_vol, vbytes) || overlaps(workspace, need, grad_out, ibytes) ||
            overlaps(workspace, need, fwd_out, ibytes) || overlaps(workspace, need, vol, sbytes) ||
            overlaps(workspace, need, Rt, (size_t)n_views * 12 * sizeof(float)))
            return fail(DRR_ERR_INVALID_ARG, "workspace overlaps another buffer");
    }
    drr::Geom g;
    drr::fill_geom(g, dims, spacing, origin, K, images, H, W, n_samples, density_factor, layout);
    g.C = channels;
    g.views_per_vol = per_vol;
    g.broadcast = bcast;
    g.vstride = stored_elements(dims, layout);
    return cuda_status(drr::launch_alpha_adjoint(vol, dtype, layout, g, Rt, grad_out, fwd_out,
                                                 grad_vol, with_ws ? workspace : nullptr,
                                                 static_cast<cudaStream_t>(stream)),
                       "drr_render_alpha_adjoint launch");
}

}  // namespace

extern "C" {

#ifdef DRR_BOUNDS_CHECK
DRR_API drr_status drr_debug_bounds_errors(unsigned long long* count, long long* first) {
    if (!count || !first) return fail(DRR_ERR_INVALID_ARG, "count and first must be non-NULL");
    cudaError_t (*const readers[])(drr::BoundsWord*) = {
        drr::bounds_word_forward, drr::bounds_word_adjoint, drr::bounds_word_pose,
        drr::bounds_word_siddon,  drr::bounds_word_prepare, drr::bounds_word_noise,
        drr::bounds_word_staged};
    *count = 0;
    *first = 0;
    for (auto read : readers) {
        drr::BoundsWord w{0ULL, 0LL};
        const cudaError_t e = read(&w);
        if (e != cudaSuccess) return cuda_status(e, "drr_debug_bounds_errors");
        if (w.count && *count == 0) *first = w.first;
        *count += w.count;
    }
    return ok();
}
#endif

DRR_API drr_status drr_wait_timeouts(unsigned long long* count) {
    if (!count) return fail(DRR_ERR_INVALID_ARG, "count must be non-NULL");
    const cudaError_t e = drr::wait_timeouts(count);
    if (e != cudaSuccess) return cuda_status(e, "drr_wait_timeouts");
    return ok();
}

DRR_API int drr_abi_version(void) { return 1; }

DRR_API const char* drr_get_last_error(void) { return g_last_error; }

DRR_API size_t drr_prepared_bytes(const int dims[3], drr_dtype dtype, drr_layout layout) {
    if (!dims) return 0;
    for (int a = 0; a < 3; ++a)
        if (dims[a] < 2 || dims[a] > kMaxDim) return 0;
    if (dtype != DRR_F32 && dtype != DRR_BF16) return 0;
    if (!known_layout(layout)) return 0;
    const int64_t n = stored_elements(dims, layout);
    if (n > kMaxElements) return 0;
    return (size_t)n * (dtype == DRR_F32 ? 4 : 2);
}

DRR_API drr_status drr_prepare_volume(const float* src, const int dims[3], drr_dtype dtype,
                                      drr_layout layout, void* dst, size_t dst_bytes,
                                      void* stream) {
    if (!dims) return fail(DRR_ERR_INVALID_ARG, "dims must be non-NULL");
    for (int a = 0; a < 3; ++a)
        if (dims[a] < 2 || dims[a] > kMaxDim)
            return fail(DRR_ERR_INVALID_ARG, "dims[%d] = %d must be in [2, %d]", a, dims[a], kMaxDim);
    if (dtype != DRR_F32 && dtype != DRR_BF16) return fail(DRR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (!known_layout(layout)) return fail(DRR_ERR_INVALID_ARG, "unknown layout %d", layout);
    const size_t need = drr_prepared_bytes(dims, dtype, layout);
    if (need == 0) return fail(DRR_ERR_UNSUPPORTED, "volume too large (max 2^31 - 1 stored elements)");
    if (!src || !dst) return fail(DRR_ERR_INVALID_ARG, "src and dst must be non-NULL");
    if (!aligned(src, 4) || !aligned(dst, layout_alignment(layout, DRR_F32)))
        return fail(DRR_ERR_INVALID_ARG, "src must be 4-byte aligned, dst 4-byte (16-byte for DRR_LAYOUT_CORNERS, _QUADS and _BRICKS)");
    if (dst_bytes < need)
        return fail(DRR_ERR_INVALID_ARG, "dst holds %zu bytes, %zu needed", dst_bytes, need);
    const size_t src_bytes = (size_t)dims[0] * dims[1] * dims[2] * 4;
    if (overlaps(src, src_bytes, dst, need)) return fail(DRR_ERR_INVALID_ARG, "src and dst overlap");
    return cuda_status(drr::launch_prepare(src, dims[0], dims[1], dims[2], dtype, layout, dst,
                                           static_cast<cudaStream_t>(stream)),
                       "drr_prepare_volume launch");
}

DRR_API drr_status drr_render(const void* vol, drr_dtype dtype, drr_layout layout,
                              const int dims[3], const float spacing[3], const float origin[3],
                              const float K[9], const float* Rt, int B, int H, int W,
                              int n_samples, float density_factor, drr_mode mode, float* out,
                              void* stream) {
    return render_batched(vol, dtype, layout, dims, spacing, origin, K, Rt, 1, 1, B, H, W,
                          n_samples, density_factor, mode, out, stream);
}

DRR_API drr_status drr_render_staged(const void* vol, drr_dtype dtype, const int dims[3],
                                     const float spacing[3], const float origin[3],
                                     const float K[9], const float* Rt, int B, int H, int W,
                                     int n_samples, float density_factor, drr_mode mode,
                                     float* out, void* stream) {
    if (mode == DRR_MODE_ALPHA)
        return fail(DRR_ERR_UNSUPPORTED,
                    "drr_render_staged integrates (raw or Beer-Lambert); alpha compositing: drr_render");
    drr_status st = check_volume(dims, spacing, origin);
    if (st != DRR_OK) return st;
    st = check_rays(K, Rt, B, H, W, n_samples, density_factor, mode);
    if (st != DRR_OK) return st;
    if (dtype != DRR_F32 && dtype != DRR_BF16) return fail(DRR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (stored_elements(dims, DRR_LAYOUT_BRICKS) > kMaxElements)
        return fail(DRR_ERR_UNSUPPORTED, "volume too large (max 2^31 - 1 stored elements)");
    if ((int64_t)B * H * W == 0) return ok();
    if (!vol || !aligned(vol, 16))
        return fail(DRR_ERR_INVALID_ARG, "vol must be a non-NULL, 16-byte aligned device pointer");
    if (!out || !aligned(out, 4))
        return fail(DRR_ERR_INVALID_ARG, "out must be a non-NULL, 4-byte aligned device pointer");
    drr::Geom g;
    drr::fill_geom(g, dims, spacing, origin, K, B, H, W, n_samples, density_factor,
                   DRR_LAYOUT_BRICKS);
    g.vstride = stored_elements(dims, DRR_LAYOUT_BRICKS);
    return cuda_status(drr::launch_forward_staged(vol, dtype, g, Rt, mode, out,
                                                  static_cast<cudaStream_t>(stream)),
                       "drr_render_staged launch");
}

DRR_API drr_status drr_render_batched(const void* vols, drr_dtype dtype, drr_layout layout,
                                      const int dims[3], const float spacing[3],
                                      const float origin[3], const float K[9], const float* Rt,
                                      int n_vols, int channels, int n_views, int H, int W,
                                      int n_samples, float density_factor, drr_mode mode,
                                      float* out, void* stream) {
    return render_batched(vols, dtype, layout, dims, spacing, origin, K, Rt, n_vols, channels,
                          n_views, H, W, n_samples, density_factor, mode, out, stream);
}

DRR_API drr_status drr_render_adjoint(const int dims[3], const float spacing[3],
                                      const float origin[3], const float K[9], const float* Rt,
                                      int B, int H, int W, int n_samples, float density_factor,
                                      drr_mode mode, const float* grad_out, const float* fwd_out,
                                      float* grad_vol, void* stream) {
    return render_adjoint_batched(dims, spacing, origin, K, Rt, 1, 1, B, H, W, n_samples,
                                  density_factor, mode, grad_out, fwd_out, grad_vol,
                                  Workspace::kNone, nullptr, 0, stream);
}

DRR_API size_t drr_adjoint_workspace_bytes(const int dims[3], int B) {
    if (!dims || B < 0 || B > kMaxViews) return 0;
    for (int a = 0; a < 3; ++a)
        if (dims[a] < 2 || dims[a] > kMaxDim) return 0;
    if (stored_elements(dims, DRR_LAYOUT_LINEAR) > kMaxElements) return 0;
    return drr::adjoint_workspace_bytes(dims[0], dims[1], dims[2], B);
}

DRR_API drr_status drr_render_adjoint_ws(const int dims[3], const float spacing[3],
                                         const float origin[3], const float K[9], const float* Rt,
                                         int B, int H, int W, int n_samples, float density_factor,
                                         drr_mode mode, const float* grad_out, const float* fwd_out,
                                         float* grad_vol, void* workspace, size_t workspace_bytes,
                                         void* stream) {
    return render_adjoint_batched(dims, spacing, origin, K, Rt, 1, 1, B, H, W, n_samples,
                                  density_factor, mode, grad_out, fwd_out, grad_vol,
                                  Workspace::kCaller, workspace, workspace_bytes, stream);
}

// Adjoint for callers that may not allocate device memory (see include/drr.h):
// the workspace of drr_render_adjoint_ws comes from the library's built-in
// scratch instead of the caller.  No allocation happens here or below.
DRR_API drr_status drr_render_adjoint_noalloc(const int dims[3], const float spacing[3],
                                              const float origin[3], const float K[9],
                                              const float* Rt, int B, int H, int W,
                                              int n_samples, float density_factor, drr_mode mode,
                                              const float* grad_out, const float* fwd_out,
                                              float* grad_vol, void* stream) {
    return render_adjoint_batched(dims, spacing, origin, K, Rt, 1, 1, B, H, W, n_samples,
                                  density_factor, mode, grad_out, fwd_out, grad_vol,
                                  Workspace::kBuiltin, nullptr, 0, stream);
}

DRR_API drr_status drr_render_adjoint_batched(const int dims[3], const float spacing[3],
                                              const float origin[3], const float K[9],
                                              const float* Rt, int n_vols, int channels,
                                              int n_views, int H, int W, int n_samples,
                                              float density_factor, drr_mode mode,
                                              const float* grad_out, const float* fwd_out,
                                              float* grad_vols, void* stream) {
    return render_adjoint_batched(dims, spacing, origin, K, Rt, n_vols, channels, n_views, H, W,
                                  n_samples, density_factor, mode, grad_out, fwd_out, grad_vols,
                                  Workspace::kNone, nullptr, 0, stream);
}

DRR_API size_t drr_adjoint_batched_workspace_bytes(const int dims[3], int n_vols, int channels,
                                                   int n_views) {
    if (!dims) return 0;
    for (int a = 0; a < 3; ++a)
        if (dims[a] < 2 || dims[a] > kMaxDim) return 0;
    if (stored_elements(dims, DRR_LAYOUT_LINEAR) > kMaxElements) return 0;
    if (n_vols < 1 || channels < 1 || n_views < 1) return 0;
    if (!(n_views == 1 || n_views % n_vols == 0)) return 0;
    const int64_t n_out = n_views == 1 ? n_vols : n_views;
    if (n_out * channels > kMaxViews) return 0;
    return drr::adjoint_workspace_bytes(dims[0], dims[1], dims[2], (int)(n_out * channels),
                                        n_vols * channels);
}

DRR_API drr_status drr_render_adjoint_batched_ws(const int dims[3], const float spacing[3],
                                                 const float origin[3], const float K[9],
                                                 const float* Rt, int n_vols, int channels,
                                                 int n_views, int H, int W, int n_samples,
                                                 float density_factor, drr_mode mode,
                                                 const float* grad_out, const float* fwd_out,
                                                 float* grad_vols, void* workspace,
                                                 size_t workspace_bytes, void* stream) {
    return render_adjoint_batched(dims, spacing, origin, K, Rt, n_vols, channels, n_views, H, W,
                                  n_samples, density_factor, mode, grad_out, fwd_out, grad_vols,
                                  Workspace::kCaller, workspace, workspace_bytes, stream);
}

DRR_API drr_status drr_render_pose_grad(const void* vol, drr_dtype dtype, drr_layout layout,
                                        const int dims[3], const float spacing[3],
                                        const float origin[3], const float K[9], const float* Rt,
                                        int B, int H, int W, int n_samples, float density_factor,
                                        drr_mode mode, const float* grad_out, const float* fwd_out,
                                        float* grad_Rt, void* stream) {
    return pose_grad_batched(vol, dtype, layout, dims, spacing, origin, K, Rt, 1, 1, B, H, W,
                             n_samples, density_factor, mode, grad_out, fwd_out, grad_Rt, stream);
}

DRR_API drr_status drr_render_pose_grad_batched(const void* vols, drr_dtype dtype,
                                                drr_layout layout, const int dims[3],
                                                const float spacing[3], const float origin[3],
                                                const float K[9], const float* Rt, int n_vols,
                                                int channels, int n_views, int H, int W,
                                                int n_samples, float density_factor,
                                                drr_mode mode, const float* grad_out,
                                                const float* fwd_out, float* grad_Rt,
                                                void* stream) {
    return pose_grad_batched(vols, dtype, layout, dims, spacing, origin, K, Rt, n_vols, channels,
                             n_views, H, W, n_samples, density_factor, mode, grad_out, fwd_out,
                             grad_Rt, stream);
}

DRR_API drr_status drr_render_alpha_adjoint(const void* vol, drr_dtype dtype, drr_layout layout,
                                            const int dims[3], const float spacing[3],
                                            const float origin[3], const float K[9],
                                            const float* Rt, int B, int H, int W, int n_samples,
                                            float density_factor, const float* grad_out,
                                            const float* fwd_out, float* grad_vol, void* stream) {
    return render_alpha_adjoint(vol, dtype, layout, dims, spacing, origin, K, Rt, 1, 1, B, H, W,
                                n_samples, density_factor, grad_out, fwd_out, grad_vol, false,
                                nullptr, 0, stream);
}

DRR_API drr_status drr_render_alpha_adjoint_ws(const void* vol, drr_dtype dtype, drr_layout layout,
                                               const int dims[3], const float spacing[3],
                                               const float origin[3], const float K[9],
                                               const float* Rt, int B, int H, int W,
                                               int n_samples, float density_factor,
                                               const float* grad_out, const float* fwd_out,
                                               float* grad_vol, void* workspace,
                                               size_t workspace_bytes, void* stream) {
    return render_alpha_adjoint(vol, dtype, layout, dims, spacing, origin, K, Rt, 1, 1, B, H, W,
                                n_samples, density_factor, grad_out, fwd_out, grad_vol, true,
                                workspace, workspace_bytes, stream);
}

DRR_API drr_status drr_render_alpha_adjoint_batched(const void* vols, drr_dtype dtype,
                                                    drr_layout layout, const int dims[3],
                                                    const float spacing[3], const float origin[3],
                                                    const float K[9], const float* Rt,
                                                    int n_vols, int channels, int n_views, int H,
                                                    int W, int n_samples, float density_factor,
                                                    const float* grad_out, const float* fwd_out,
                                                    float* grad_vols, void* workspace,
                                                    size_t workspace_bytes, void* stream) {
    return render_alpha_adjoint(vols, dtype, layout, dims, spacing, origin, K, Rt, n_vols,
                                channels, n_views, H, W, n_samples, density_factor, grad_out,
                                fwd_out, grad_vols, workspace != nullptr, workspace,
                                workspace_bytes, stream);
}

DRR_API drr_status drr_poisson_noise(const float* image, const float* z, float i0, float* out,
                                     int64_t n, void* stream) {
    if (!(i0 > 0.0f) || !std::isfinite(i0))
        return fail(DRR_ERR_INVALID_ARG, "i0 must be finite and > 0");
    if (n < 0) return fail(DRR_ERR_INVALID_ARG, "n must be >= 0");
    if (n == 0) return ok();
    if (!image || !z || !out || !aligned(image, 4) || !aligned(z, 4) || !aligned(out, 4))
        return fail(DRR_ERR_INVALID_ARG, "image, z and out must be non-NULL, 4-byte aligned device pointers");
    const size_t bytes = (size_t)n * 4;
    if ((out != image && overlaps(out, bytes, image, bytes)) || overlaps(out, bytes, z, bytes))
        return fail(DRR_ERR_INVALID_ARG, "out overlaps z or part of image (it may be image itself)");
    return cuda_status(drr::launch_poisson_noise(image, z, i0, out, n, static_cast<cudaStream_t>(stream)),
                       "drr_poisson_noise launch");
}

DRR_API drr_status drr_poisson_noise_backward(const float* image, const float* z, float i0,
                                              const float* grad_out, float* grad_image, int64_t n,
                                              void* stream) {
    if (!(i0 > 0.0f) || !std::isfinite(i0))
        return fail(DRR_ERR_INVALID_ARG, "i0 must be finite and > 0");
    if (n < 0) return fail(DRR_ERR_INVALID_ARG, "n must be >= 0");
    if (n == 0) return ok();
    if (!image || !z || !grad_out || !grad_image || !aligned(image, 4) || !aligned(z, 4) ||
        !aligned(grad_out, 4) || !aligned(grad_image, 4))
        return fail(DRR_ERR_INVALID_ARG,
                    "image, z, grad_out and grad_image must be non-NULL, 4-byte aligned device pointers");
    const size_t bytes = (size_t)n * 4;
    if (overlaps(grad_image, bytes, image, bytes) || overlaps(grad_image, bytes, z, bytes) ||
        (grad_image != grad_out && overlaps(grad_image, bytes, grad_out, bytes)))
        return fail(DRR_ERR_INVALID_ARG, "grad_image overlaps image, z or part of grad_out");
    return cuda_status(drr::launch_poisson_noise_backward(image, z, i0, grad_out, grad_image, n,
                                                          static_cast<cudaStream_t>(stream)),
                       "drr_poisson_noise_backward launch");
}

DRR_API drr_status drr_render_siddon(const void* vol, drr_dtype dtype, const int dims[3],
                                     const float spacing[3], const float origin[3],
                                     const float K[9], const float* Rt, int B, int H, int W,
                                     float density_factor, drr_mode mode, float* out,
                                     void* stream) {
    if (mode == DRR_MODE_ALPHA)
        return fail(DRR_ERR_UNSUPPORTED, "the cell-constant projector writes DRR_MODE_RAW or DRR_MODE_BEER_LAMBERT");
    drr_status st = check_volume(dims, spacing, origin);
    if (st != DRR_OK) return st;
    st = check_rays(K, Rt, B, H, W, 1, density_factor, mode);
    if (st != DRR_OK) return st;
    if (dtype != DRR_F32 && dtype != DRR_BF16) return fail(DRR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (stored_elements(dims, DRR_LAYOUT_LINEAR) > kMaxElements)
        return fail(DRR_ERR_UNSUPPORTED, "volume too large (max 2^31 - 1 elements)");
    if ((int64_t)B * H * W == 0) return ok();
    if (!vol || !aligned(vol, dtype == DRR_F32 ? 4 : 2))
        return fail(DRR_ERR_INVALID_ARG, "vol must be a non-NULL, aligned device pointer");
    if (!out || !aligned(out, 4)) return fail(DRR_ERR_INVALID_ARG, "out must be a non-NULL, 4-byte aligned device pointer");
    drr::Geom g;
    drr::fill_geom(g, dims, spacing, origin, K, B, H, W, 1, density_factor, DRR_LAYOUT_LINEAR);
    return cuda_status(drr::launch_siddon(vol, dtype, g, Rt, mode, out, static_cast<cudaStream_t>(stream)),
                       "drr_render_siddon launch");
}

DRR_API drr_status drr_render_siddon_adjoint(const int dims[3], const float spacing[3],
                                             const float origin[3], const float K[9],
                                             const float* Rt, int B, int H, int W,
                                             float density_factor, drr_mode mode,
                                             const float* grad_out, const float* fwd_out,
                                             float* grad_vol, void* stream) {
    if (mode == DRR_MODE_ALPHA)
        return fail(DRR_ERR_UNSUPPORTED, "the cell-constant projector writes DRR_MODE_RAW or DRR_MODE_BEER_LAMBERT");
    drr_status st = check_volume(dims, spacing, origin);
    if (st != DRR_OK) return st;
    st = check_rays(K, Rt, B, H, W, 1, density_factor, mode);
    if (st != DRR_OK) return st;
    if (stored_elements(dims, DRR_LAYOUT_LINEAR) > kMaxElements)
        return fail(DRR_ERR_UNSUPPORTED, "volume too large (max 2^31 - 1 elements)");
    const int64_t npix = (int64_t)B * H * W;
    if (npix == 0) return ok();
    if (!grad_out || !aligned(grad_out, 4))
        return fail(DRR_ERR_INVALID_ARG, "grad_out must be a non-NULL, 4-byte aligned device pointer");
    if (mode == DRR_MODE_BEER_LAMBERT && (!fwd_out || !aligned(fwd_out, 4)))
        return fail(DRR_ERR_INVALID_ARG, "fwd_out is required in Beer-Lambert mode");
    if (!grad_vol || !aligned(grad_vol, 4))
        return fail(DRR_ERR_INVALID_ARG, "grad_vol must be a non-NULL, 4-byte aligned device pointer");
    const size_t vbytes = (size_t)dims[0] * dims[1] * dims[2] * 4, ibytes = (size_t)npix * 4;
    if (overlaps(grad_vol, vbytes, grad_out, ibytes) ||
        (mode == DRR_MODE_BEER_LAMBERT && overlaps(grad_vol, vbytes, fwd_out, ibytes)))
        return fail(DRR_ERR_INVALID_ARG, "grad_vol overlaps an image buffer");
    drr::Geom g;
    drr::fill_geom(g, dims, spacing, origin, K, B, H, W, 1, density_factor, DRR_LAYOUT_LINEAR);
    return cuda_status(drr::launch_siddon_adjoint(g, Rt, mode, grad_out, fwd_out, grad_vol,
                                                  static_cast<cudaStream_t>(stream)),
                       "drr_render_siddon_adjoint launch");
}

}  // extern "C"

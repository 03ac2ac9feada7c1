// drr_internal.cuh -- device-side geometry shared by the forward and adjoint
// kernels of libdrr (per-view setup, per-ray setup and slab clip).
//
// The method (see include/drr.h): Hartley-Zisserman pinhole rays (nanodrr
// page, introduction), clipped to the volume box (flashdrr.rendering API
// docs, compute_clipping_distances) with the slab method, sampled with the
// midpoint rule and zero-padded trilinear interpolation in IJK space
// (VolumeRaycaster.forward / __init__: ray_samples, density_factor).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace drr {

// Launch shape of every ray kernel: a CTA renders a 16 x 16 pixel tile of one
// view; each warp owns an 8 x 4 sub-tile so that its 32 rays are spatial
// neighbours and their trilinear footprints share cache lines.
constexpr int kTileW = 16;
constexpr int kTileH = 16;
constexpr int kThreads = kTileW * kTileH;
constexpr int kWarpW = 8;
constexpr int kWarpH = 4;

// Everything a ray kernel needs besides the device pointers; passed by value.
struct Geom {
    int nx, ny, nz;          // logical volume dims
    int row, slice;          // element strides of j and k in the stored layout
    float hi[3];             // n - 1 per axis: the voxel-centre box is [0, hi]
    long long lim[3];        // largest 32.32 sample coordinate the stored layout allows
    double spacing[3];       // voxel size, mm
    double origin[3];        // world mm of voxel 0's centre
    double kinv[6];          // K^-1 = [k0 k1 k2; 0 k3 k4; 0 0 k5], from fp64 on the host
    int B, H, W, N;
    float density_factor;
    // Batches of volumes and channels (VolumeRaycaster.forward's (B, C, D,
    // H, W) volumes and N = B * views_per_vol view matrices, N == 1
    // broadcast): grid z = output view n times C plus channel ch; view n
    // uses pose n (pose 0 when broadcast) and volume n / views_per_vol
    // (volume n when broadcast); volume v, channel ch starts vstride
    // elements after the previous one.  One volume of one channel: C = 1,
    // views_per_vol = B, no broadcast.
    int C;
    int views_per_vol;
    int broadcast;
    long long vstride;
};

// Pose, volume-channel slot and output image of grid z.
struct BatchItem {
    int pose;         // row of Rt
    long long slot;   // volume * C + channel
};

// Number of volume-channel slots a batched call touches.
__host__ __device__ __forceinline__ int batch_slots(const Geom& g) {
    const int n_out = g.B / g.C;
    return (g.broadcast ? n_out : n_out / g.views_per_vol) * g.C;
}

__device__ __forceinline__ BatchItem batch_item(const Geom& g, int z) {
    const int n = z / g.C, ch = z - n * g.C;
    BatchItem it;
    it.pose = g.broadcast ? 0 : n;
    const int v = g.broadcast ? n : n / g.views_per_vol;
    it.slot = (long long)v * g.C + ch;
    return it;
}

// Per-view quantities, computed once per CTA from the view's [R|t], in fp64
// (the pose is widened from fp32; the camera sits hundreds of voxels from
// the volume, so fp32 here would cost ~1e-4 voxel of sample position):
//   A = R^T K^-1  (pixel (u, v, 1) -> world direction, unnormalised)
//   C = (-R^T t - origin) / spacing  (camera centre in IJK)
struct View {
    double A[9];
    double C[3];
};

__device__ __forceinline__ void view_setup(const float* __restrict__ Rt12, const Geom& g,
                                           View& v) {
    double R[9], t[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
#pragma unroll
        for (int c = 0; c < 3; ++c) R[3 * r + c] = (double)Rt12[4 * r + c];
        t[r] = (double)Rt12[4 * r + 3];
    }
    const double i00 = g.kinv[0], i01 = g.kinv[1], i02 = g.kinv[2];
    const double i11 = g.kinv[3], i12 = g.kinv[4], i22 = g.kinv[5];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        // column a of R is row a of R^T
        const double r0 = R[a], r1 = R[3 + a], r2 = R[6 + a];
        v.A[3 * a + 0] = r0 * i00;
        v.A[3 * a + 1] = r0 * i01 + r1 * i11;
        v.A[3 * a + 2] = r0 * i02 + r1 * i12 + r2 * i22;
        const double cw = -(r0 * t[0] + r1 * t[1] + r2 * t[2]);
        v.C[a] = (cw - g.origin[a]) / g.spacing[a];
    }
}

// One ray, clipped and discretised.  Sample positions are 32.32 fixed point
// per axis (high word: the cell index, low word: the fraction), advanced by
// exact integer adds: sample i sits at q0 + i * s.  An fp32 position would
// carry ~1e-5 voxel of rounding at coordinates ~256, which a ray grazing a
// sharp edge turns into ~1e-4 of its integral; here the positions are exact
// to ~1e-9 voxel and the fraction handed to the interpolation to 2^-23.
// Because positions are exactly linear in i, keeping the first and the last
// sample inside [0, lim] keeps every sample inside: that is the whole memory-
// safety argument of the sample loops.
struct Ray {
    long long q0[3];
    long long s[3];
    float dt;
};

constexpr double kFix = 4294967296.0;           // 2^32

// fraction of a 32.32 coordinate as a float in [0, 1), from its top 23 bits
__device__ __forceinline__ float fix_frac(long long q) {
    const unsigned lo = (unsigned)(unsigned long long)q;
    return __uint_as_float(0x3F800000u | (lo >> 9)) - 1.0f;
}

// The same value another way: a funnel shift of the pair (0x7F : lo) right
// by 9 leaves lo's top 23 bits as a mantissa under the exponent of 1.0 (the
// float 1 + f in one instruction), then the exact subtraction.  Bit for bit
// fix_frac; which runs faster depends on the loop around it (B200: the
// xy-quad forward 8-16 % and the brick forward 3 % faster with this one, the
// corner-record forward 2-22 % and the record adjoint 1 % slower), so each
// loop uses the one measured faster.
__device__ __forceinline__ float fix_frac_fs(long long q) {
    const unsigned lo = (unsigned)(unsigned long long)q;
    return __uint_as_float(__funnelshift_r(lo, 0x7Fu, 9)) - 1.0f;
}

__device__ __forceinline__ int fix_cell(long long q) { return (int)(q >> 32); }

// Returns false for a miss (or a ray whose geometry is not finite).
//   offset     added to the IJK coordinates (1 for the zero-bordered layout)
//   g.lim[k]   largest allowed 32.32 coordinate along axis k; the smallest is
//              0.  Samples that rounding pushes past [0, lim] are pulled back
//              by a few 2^-32 voxel.
__device__ __forceinline__ bool ray_setup(const View& v, const Geom& g, double u, double w,
                                          double offset, Ray& ray) {
    double a[3], d[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) a[k] = v.A[3 * k] * u + v.A[3 * k + 1] * w + v.A[3 * k + 2];
    const double rn = 1.0 / sqrt(a[0] * a[0] + a[1] * a[1] + a[2] * a[2]);
    double t_near = -INFINITY, t_far = INFINITY;
    bool ok = true;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        d[k] = a[k] * rn / g.spacing[k];
        const double c = v.C[k];
        ok = ok && isfinite(d[k]) && isfinite(c);
        if (d[k] != 0.0) {
            const double ta = (0.0 - c) / d[k];
            const double tb = ((double)g.hi[k] - c) / d[k];
            t_near = fmax(t_near, fmin(ta, tb));
            t_far = fmin(t_far, fmax(ta, tb));
        } else {
            // parallel to this slab: inside (planes included) or a miss
            ok = ok && (c >= 0.0) && (c <= (double)g.hi[k]);
        }
    }
    const double t0 = fmax(t_near, 0.0);
    const double t1 = t_far;
    if (!ok || !(t1 > t0) || !isfinite(t1)) return false;
    const double dt = (t1 - t0) / (double)g.N;
    const double tm = t0 + 0.5 * dt;                 // parameter of sample 0
    const long long last = g.N - 1;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const double first_d = v.C[k] + tm * d[k] + offset;
        const double end_d = first_d + (double)last * dt * d[k];
        // inside the box these are < 2^22; anything far outside is absurd geometry
        if (!(fabs(first_d) < 16777216.0 && fabs(end_d) < 16777216.0)) return false;
        // + 2^8: fix_frac truncates to 23 bits, so this makes it round to nearest
        long long first = __double2ll_rn(first_d * kFix) + 256;
        long long step = __double2ll_rn(dt * d[k] * kFix);
        long long end = first + last * step;
        const long long lim = g.lim[k];
        if (first < 0 || first > lim || end < 0 || end > lim) {
            first = min(max(first, 0LL), lim);
            end = min(max(end, 0LL), lim);
            step = last > 0 ? (end - first) / last : 0;   // truncation keeps q0 + last*s in range
        }
        ray.q0[k] = first;
        ray.s[k] = step;
    }
    ray.dt = (float)dt;
    return true;
}

// ---------------------------------------------------------------------------
// Bounds-checked debug build.  Compiled with -DDRR_BOUNDS_CHECK (into
// libdrr_checked.so), every gather and scatter of the kernels tests its
// element range [off, off + len) against the extent n of the buffer (or of
// the volume-channel slot) it addresses; an access outside is skipped (a
// load reads 0) and counted in this translation unit's error word, with the
// first offending offset.  drr_debug_bounds_errors (include/drr_debug.h)
// reads and clears the words of every unit.  In the ordinary build the test
// is the constant true and compiles away.
struct BoundsWord {
    unsigned long long count;
    long long first;
};

#ifdef DRR_BOUNDS_CHECK
static __device__ BoundsWord g_bounds_word;

__device__ __forceinline__ bool in_bounds(long long off, long long len, long long n) {
    if (off >= 0 && len >= 0 && off <= n - len) return true;
    if (atomicAdd(&g_bounds_word.count, 1ULL) == 0ULL) g_bounds_word.first = off;
    return false;
}

// Host: this unit's error word (read, then cleared); defined once per .cu
// file that launches kernels, under the given name.
#define DRR_BOUNDS_READER(name)                                                  \
    cudaError_t name(BoundsWord* out) {                                          \
        cudaError_t e = cudaMemcpyFromSymbol(out, g_bounds_word, sizeof(*out));  \
        if (e != cudaSuccess) return e;                                          \
        const BoundsWord zero{0ULL, 0LL};                                        \
        return cudaMemcpyToSymbol(g_bounds_word, &zero, sizeof(zero));           \
    }
#else
__device__ __forceinline__ constexpr bool in_bounds(long long, long long, long long) {
    return true;
}
#define DRR_BOUNDS_READER(name)
#endif

// Bricked layout (4): the cells in bricks of kBrick^3; brick (bx, by, bz)
// stores the voxels (kBrick bx + lx, kBrick by + ly, kBrick bz + lz) for lx,
// ly, lz in [0, kBrick] -- its cells' corners, the last plane of each axis
// shared with the next brick (a one-voxel apron) -- x fastest, padded to
// kBrickStride elements (a multiple of 16 bytes for fp32 and bf16).  A cell's
// 8 corners then lie in one brick, at the constant offsets a + kBrickEdge b
// + kBrickPlane c, and a brick (2.9 KB fp32) is one contiguous block.  Brick
// (bx, by, bz) is number (bz * nby + by) * nbx + bx; in Geom, row = nbx and
// slice = nbx * nby.
constexpr int kBrick = 8;
constexpr int kBrickEdge = kBrick + 1;
constexpr int kBrickPlane = kBrickEdge * kBrickEdge;
constexpr int kBrickStride = 736;          // 729 voxels, padded
static_assert(kBrickStride >= kBrickPlane * kBrickEdge && kBrickStride % 8 == 0, "brick stride");

// bricks along an axis of n voxels (n - 1 cells)
__host__ __device__ __forceinline__ int brick_count(int n) { return (n - 1 + kBrick - 1) / kBrick; }

// element of corner (0, 0, 0) of cell (cx, cy, cz) in the bricked layout
__device__ __forceinline__ int brick_element(const Geom& g, int cx, int cy, int cz) {
    const int brick = (cz >> 3) * g.slice + (cy >> 3) * g.row + (cx >> 3);
    const int local = ((cz & 7) * kBrickEdge + (cy & 7)) * kBrickEdge + (cx & 7);
    return brick * kBrickStride + local;
}
static_assert(kBrick == 8, "brick_element shifts by 3");

// Index of cell (cx, cy, cz) in each stored layout (0 linear, 1 zero-bordered,
// 2 corner records, 3 xy quads, 4 bricks): a cell, record or quad number,
// or for bricks the element of its first corner.
template <int LAYOUT>
__device__ __forceinline__ int cell_index(const Geom& g, int cx, int cy, int cz) {
    if constexpr (LAYOUT == 4) return brick_element(g, cx, cy, cz);
    return cz * g.slice + cy * g.row + cx;
}

// Elements one trilinear sample reads, from the offset of its cell's first
// element, in each stored layout, and that offset for cell index `cell`.
template <int LAYOUT>
__host__ __device__ __forceinline__ long long sample_extent(const Geom& g) {
    return LAYOUT == 2   ? 8
           : LAYOUT == 3 ? 4LL * g.slice + 4
           : LAYOUT == 4 ? (long long)kBrickPlane + kBrickEdge + 2
                         : (long long)g.slice + g.row + 2;
}
template <int LAYOUT>
__host__ __device__ __forceinline__ long long sample_offset(long long cell) {
    return LAYOUT == 2 ? cell * 8 : LAYOUT == 3 ? cell * 4 : cell;
}

// Pixel of this thread inside a kTileW x kTileH tile (warps are 8 x 4).
__device__ __forceinline__ void tile_pixel(int& r, int& c) {
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    constexpr int warps_per_row = kTileW / kWarpW;
    const int wx = warp % warps_per_row, wy = warp / warps_per_row;
    c = blockIdx.x * kTileW + wx * kWarpW + (lane % kWarpW);
    r = blockIdx.y * kTileH + wy * kWarpH + (lane / kWarpW);
}

// ---------------------------------------------------------------------------
// host side

// Kernel parameter block from validated host arguments.  layout: 0 linear,
// 1 zero-bordered, 2 corner records, 3 xy quads, 4 bricks (include/drr.h).  K^-1 of the upper
// triangular K in double.
inline void fill_geom(Geom& g, const int dims[3], const float spacing[3], const float origin[3],
                      const float K[9], int B, int H, int W, int n_samples, float density_factor,
                      int layout) {
    g = Geom{};
    g.nx = dims[0];
    g.ny = dims[1];
    g.nz = dims[2];
    if (layout == 2 || layout == 3) {       // strides of cells (8 elements) or quads (4)
        g.row = dims[0] - 1;
        g.slice = (dims[0] - 1) * (dims[1] - 1);
    } else if (layout == 4) {               // bricks per row and per slice of bricks
        g.row = brick_count(dims[0]);
        g.slice = brick_count(dims[0]) * brick_count(dims[1]);
    } else {
        const int pad = layout == 1 ? 2 : 0;
        g.row = dims[0] + pad;
        g.slice = (dims[0] + pad) * (dims[1] + pad);
    }
    for (int a = 0; a < 3; ++a) {
        g.hi[a] = (float)(dims[a] - 1);
        // largest 32.32 sample coordinate whose 8 corners are stored: cell <= n-2
        // for the linear, corner and quad layouts, cell <= n (inside the zero
        // border) for the bordered one
        const long long cells = layout == 1 ? dims[a] + 1 : dims[a] - 1;
        g.lim[a] = cells * (1LL << 32) - 1;
        g.spacing[a] = spacing[a];
        g.origin[a] = origin[a];
    }
    const double k0 = K[0], k1 = K[1], k2 = K[2], k4 = K[4], k5 = K[5], k8 = K[8];
    g.kinv[0] = 1.0 / k0;
    g.kinv[1] = -k1 / (k0 * k4);
    g.kinv[2] = (k1 * k5 - k2 * k4) / (k0 * k4 * k8);
    g.kinv[3] = 1.0 / k4;
    g.kinv[4] = -k5 / (k4 * k8);
    g.kinv[5] = 1.0 / k8;
    g.B = B;
    g.H = H;
    g.W = W;
    g.N = n_samples;
    g.density_factor = density_factor;
    g.C = 1;
    g.views_per_vol = B > 0 ? B : 1;
    g.broadcast = 0;
    g.vstride = 0;
}

// launchers (defined in the .cu files)

cudaError_t launch_forward(const void* vol, int dtype, int layout, const Geom& g,
                           const float* Rt, int mode, float* out, cudaStream_t stream);
// the bricked layout's forward with each frustum layer's bricks staged in
// shared memory by bulk copies (drr_staged.cu; raw and Beer-Lambert modes)
cudaError_t launch_forward_staged(const void* vol, int dtype, const Geom& g, const float* Rt,
                                  int mode, float* out, cudaStream_t stream);
cudaError_t launch_adjoint(const Geom& g, const float* Rt, int mode, const float* grad_out,
                           const float* fwd_out, float* grad_vol, void* workspace,
                           cudaStream_t stream);
size_t adjoint_workspace_bytes(int nx, int ny, int nz, int B, int slots = 1);

// Size of the built-in scratch of the allocation-free adjoint (32 MiB).
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
// Device address of that scratch on the current device (drr_adjoint.cu),
// looked up once per device and cached for the life of the process.
cudaError_t noalloc_scratch(void** out);
// Grid-barrier waits of the adjoint's slab pass that gave up, on the current
// device, since the last read (drr_adjoint.cu); the count is cleared.
cudaError_t wait_timeouts(unsigned long long* out);
cudaError_t launch_prepare(const float* src, int nx, int ny, int nz, int dtype, int layout,
                           void* dst, cudaStream_t stream);
// workspace: NULL (every view on the direct path) or the layout of
// adjoint_workspace_bytes (dense views accumulate into corner records)
cudaError_t launch_alpha_adjoint(const void* vol, int dtype, int layout, const Geom& g,
                                 const float* Rt, const float* grad_out, const float* fwd_out,
                                 float* grad_vol, void* workspace, cudaStream_t stream);
cudaError_t launch_poisson_noise(const float* image, const float* z, float i0, float* out,
                                 int64_t n, cudaStream_t stream);
cudaError_t launch_poisson_noise_backward(const float* image, const float* z, float i0,
                                          const float* grad_out, float* grad_image, int64_t n,
                                          cudaStream_t stream);
cudaError_t launch_siddon(const void* vol, int dtype, const Geom& g, const float* Rt, int mode,
                          float* out, cudaStream_t stream);
cudaError_t launch_siddon_adjoint(const Geom& g, const float* Rt, int mode, const float* grad_out,
                                  const float* fwd_out, float* grad_vol, cudaStream_t stream);
// per-unit readers of the bounds-check error words (the checked build only)
#ifdef DRR_BOUNDS_CHECK
cudaError_t bounds_word_forward(BoundsWord* out);
cudaError_t bounds_word_adjoint(BoundsWord* out);
cudaError_t bounds_word_pose(BoundsWord* out);
cudaError_t bounds_word_siddon(BoundsWord* out);
cudaError_t bounds_word_prepare(BoundsWord* out);
cudaError_t bounds_word_noise(BoundsWord* out);
cudaError_t bounds_word_staged(BoundsWord* out);
#endif

cudaError_t launch_pose_grad(const void* vol, int dtype, int layout, const Geom& g,
                             const float* Rt, int mode, const float* grad_out,
                             const float* fwd_out, float* grad_Rt, cudaStream_t stream);

}  // namespace drr

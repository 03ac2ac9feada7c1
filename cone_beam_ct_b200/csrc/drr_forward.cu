// drr_forward.cu -- forward DRR ray-march kernels (sm_100a).
//
// One thread per ray, a 16 x 16 pixel tile per CTA (warps own 8 x 4
// sub-tiles).  Per ray: view/ray setup and slab clip (drr_internal.cuh),
// then n_samples midpoint samples of the zero-padded trilinear interpolant,
// summed in fp32, then I = density_factor * dt * sum written raw or as
// 1 - exp(-I) (flashdrr.rendering API docs, VolumeRaycaster.__init__:
// ray_samples, density_factor, use_beer_lambert), or composited front to
// back (use_beer_lambert = False; march_alpha below).  Nothing per sample is
// materialised in memory: the fused design the FlashDRR page credits for its
// near-constant footprint ("Memory Scaling").
//
// Four storage layouts (include/drr.h): the caller's linear array, the
// array inside a one-voxel zero border, corner records or xy quads
// (drr_sample.cuh reads one sample from each).  Sample positions are
// 32.32 fixed point (drr_internal.cuh), clipped per ray so that every corner
// read stays inside the stored volume; inside the voxel-centre box the linear
// layout's upper corner at n-1 is reached with weight 1 - 2^-32 instead of
// through the border, an O(2^-32) difference.
#include <cuda_runtime.h>
#include <stdint.h>

#include "drr_internal.cuh"
#include "drr_sample.cuh"

namespace drr {
namespace {

// Sum of the N samples of one ray.  Every sample lies in [0, g.lim] per axis
// (ray_setup), so the 8 corners of every sample lie inside the stored volume:
// for the linear layout lim < (n-1) * 2^32 (cell <= n-2), for the padded one
// lim < (n+1) * 2^32 (cell <= n, inside the zero border).
template <typename T>
__device__ __forceinline__ float march(const T* __restrict__ vol, const Geom& g, const Ray& ray) {
    const int row = g.row, slice = g.slice;
    long long qx = ray.q0[0], qy = ray.q0[1], qz = ray.q0[2];
    const long long sx = ray.s[0], sy = ray.s[1], sz = ray.s[2];
    float acc = 0.0f;
#pragma unroll 4
    for (int i = 0; i < g.N; ++i) {
        const int idx = fix_cell(qz) * slice + fix_cell(qy) * row + fix_cell(qx);
        if (in_bounds(idx, sample_extent<0>(g), g.vstride))
            acc += trilinear_at(vol + idx, row, slice, fix_frac(qx), fix_frac(qy), fix_frac(qz));
        qx += sx;
        qy += sy;
        qz += sz;
    }
    return acc;
}

// Unroll of the corner-layout sample loop: the largest that ptxas compiles
// without spilling for each element type under the kernel's launch bounds.
template <typename T>
constexpr int kCornerUnroll = sizeof(T) == 2 ? 2 : 4;

// Sum of the N samples of one ray in the corner-replicated layout: one cell
// record per sample.  Cells stay in [0, n-2] (g.lim as for the linear
// layout), inside the stored records.
template <typename T>
__device__ __forceinline__ float march_corners(const T* __restrict__ vol, const Geom& g,
                                               const Ray& ray) {
    const int row = g.row, slice = g.slice;      // cell strides
    long long qx = ray.q0[0], qy = ray.q0[1], qz = ray.q0[2];
    const long long sx = ray.s[0], sy = ray.s[1], sz = ray.s[2];
    float acc = 0.0f;
#pragma unroll(kCornerUnroll<T>)
    for (int i = 0; i < g.N; ++i) {
        const int cell = fix_cell(qz) * slice + fix_cell(qy) * row + fix_cell(qx);
        if (in_bounds(sample_offset<2>(cell), 8, g.vstride))
            acc += sample_corners(vol + (size_t)cell * 8, fix_frac(qx), fix_frac(qy), fix_frac(qz));
        qx += sx;
        qy += sy;
        qz += sz;
    }
    return acc;
}

// Sum of the N samples of one ray in the bricked layout: one brick per
// sample, its 8 corners at constant offsets.  Cells stay in [0, n-2] (g.lim
// as for the linear layout), inside the stored bricks.
template <typename T>
__device__ __forceinline__ float march_bricks(const T* __restrict__ vol, const Geom& g,
                                              const Ray& ray) {
    long long qx = ray.q0[0], qy = ray.q0[1], qz = ray.q0[2];
    const long long sx = ray.s[0], sy = ray.s[1], sz = ray.s[2];
    float acc = 0.0f;
#pragma unroll 4
    for (int i = 0; i < g.N; ++i) {
        const int e = brick_element(g, fix_cell(qx), fix_cell(qy), fix_cell(qz));
        if (in_bounds(e, sample_extent<4>(g), g.vstride))
            acc += sample_brick(vol + e, fix_frac_fs(qx), fix_frac_fs(qy), fix_frac_fs(qz));
        qx += sx;
        qy += sy;
        qz += sz;
    }
    return acc;
}

// Front-to-back alpha compositing of one ray (the over operator; flashdrr
// rendering API docs, VolumeRaycaster.__init__, use_beer_lambert = False),
// read as the emission-absorption sum: sample i has opacity
// a_i = 1 - exp(-s mu_i), s = density_factor * dt, and colour mu_i;
// C = sum_i T_i a_i mu_i with T_0 = 1, T_{i+1} = T_i (1 - a_i).  The same
// samples and interpolation as the integral; a_i by opacity<T>
// (drr_sample.cuh), which keeps its relative accuracy for the small
// opacities of thin samples.
template <typename T, int LAYOUT>
__device__ __forceinline__ float march_alpha(const T* __restrict__ vol, const Geom& g,
                                             const Ray& ray, float s) {
    const int row = g.row, slice = g.slice;
    long long qx = ray.q0[0], qy = ray.q0[1], qz = ray.q0[2];
    const long long sx = ray.s[0], sy = ray.s[1], sz = ray.s[2];
    float C = 0.0f, Tr = 1.0f;
    for (int i = 0; i < g.N; ++i) {
        const int cell = cell_index<LAYOUT>(g, fix_cell(qx), fix_cell(qy), fix_cell(qz));
        const float fx = fix_frac(qx), fy = fix_frac(qy), fz = fix_frac(qz);
        const float mu =
            !in_bounds(sample_offset<LAYOUT>(cell), sample_extent<LAYOUT>(g), g.vstride) ? 0.0f
            : LAYOUT == 4 ? sample_brick(vol + cell, fx, fy, fz)
            : LAYOUT == 2 ? sample_corners(vol + (size_t)cell * 8, fx, fy, fz)
            : LAYOUT == 3 ? sample_quads(vol + (size_t)cell * 4, slice, fx, fy, fz)
                          : trilinear_at(vol + cell, row, slice, fx, fy, fz);
        const float a = opacity<T>(s * mu);
        C = fmaf(Tr * a, mu, C);
        Tr *= 1.0f - a;
        qx += sx;
        qy += sy;
        qz += sz;
    }
    return C;
}

// Sum of the N samples of one ray in the xy-quad layout: two quads per
// sample.  Quads stay in [0, n-2] x [0, n-2] x [0, n-2] (g.lim as for the
// linear layout), so both slices read are stored.  Measured on B200 for the
// 256^3 fp32 volume seen by 64 views of 200^2: 2.18 ms against 2.89 for
// corner records (half the footprint: less of it re-read from DRAM) and 2.44
// for x pairs; for the 512^3 fp32 volume seen by 2 views of 2048^2, whose
// dense rays reuse records in L1, corner records stay faster (4.0 against
// 4.5 ms).
template <typename T>
__device__ __forceinline__ float march_quads(const T* __restrict__ vol, const Geom& g,
                                             const Ray& ray) {
    const int row = g.row, slice = g.slice;      // quad strides
    long long qx = ray.q0[0], qy = ray.q0[1], qz = ray.q0[2];
    const long long sx = ray.s[0], sy = ray.s[1], sz = ray.s[2];
    float acc = 0.0f;
#pragma unroll 4
    for (int i = 0; i < g.N; ++i) {
        const int q = fix_cell(qz) * slice + fix_cell(qy) * row + fix_cell(qx);
        if (in_bounds(sample_offset<3>(q), sample_extent<3>(g), g.vstride))
            acc += sample_quads(vol + (size_t)q * 4, slice, fix_frac_fs(qx), fix_frac_fs(qy),
                                fix_frac_fs(qz));
        qx += sx;
        qy += sy;
        qz += sz;
    }
    return acc;
}

// CTAs per SM the compiler must fit: 5 for bf16 corner records (at most 51
// registers; B200, 1024^2 x 512 C-arm views: 2.80 against 2.86 ms), no
// minimum (0) for the rest (the fp32 quad forward ran 2-7 % slower when held
// to 5 or 6)
template <typename T, int LAYOUT>
constexpr int kForwardMinBlocks = (sizeof(T) == 2 && LAYOUT == 2) ? 5 : 0;

template <typename T, int LAYOUT, int MODE>
__global__ void __launch_bounds__(kThreads, (kForwardMinBlocks<T, LAYOUT>))
forward_kernel(const T* __restrict__ vol_base, const float* __restrict__ Rt,
               float* __restrict__ out, const Geom g) {
    __shared__ View sv;
    const int b = blockIdx.z;                    // output image (view x channel)
    const BatchItem it = batch_item(g, b);
    const T* __restrict__ vol = vol_base + it.slot * g.vstride;
    if (!in_bounds(it.slot * g.vstride, g.vstride, batch_slots(g) * g.vstride)) return;
    if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)it.pose, g, sv);
    __syncthreads();
    int r, c;
    tile_pixel(r, c);
    if (r >= g.H || c >= g.W) return;
    Ray ray;
    float result = 0.0f;
    if (ray_setup(sv, g, (double)c, (double)r, LAYOUT == 1 ? 1.0 : 0.0, ray)) {
        if (MODE == 2) {
            result = march_alpha<T, LAYOUT>(vol, g, ray, g.density_factor * ray.dt);
        } else {
            const float sum = LAYOUT == 2   ? march_corners(vol, g, ray)
                              : LAYOUT == 3 ? march_quads(vol, g, ray)
                              : LAYOUT == 4 ? march_bricks(vol, g, ray)
                                            : march(vol, g, ray);
            const float I = (g.density_factor * ray.dt) * sum;
            result = (MODE == 1) ? -expm1f(-I) : I;
        }
    }
    const long long pix = ((long long)b * g.H + r) * g.W + c;
    if (in_bounds(pix, 1, (long long)g.B * g.H * g.W)) out[pix] = result;
}

template <typename T, int LAYOUT>
cudaError_t launch_typed(const void* vol, const Geom& g, const float* Rt, int mode, float* out,
                         cudaStream_t stream) {
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    const T* v = static_cast<const T*>(vol);
    if (mode == 2)
        forward_kernel<T, LAYOUT, 2><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    else if (mode == 1)
        forward_kernel<T, LAYOUT, 1><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    else
        forward_kernel<T, LAYOUT, 0><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_layout(const void* vol, int layout, const Geom& g, const float* Rt, int mode,
                          float* out, cudaStream_t stream) {
    if (layout == 4) return launch_typed<T, 4>(vol, g, Rt, mode, out, stream);
    if (layout == 3) return launch_typed<T, 3>(vol, g, Rt, mode, out, stream);
    if (layout == 2) return launch_typed<T, 2>(vol, g, Rt, mode, out, stream);
    if (layout == 1) return launch_typed<T, 1>(vol, g, Rt, mode, out, stream);
    return launch_typed<T, 0>(vol, g, Rt, mode, out, stream);
}

}  // namespace

DRR_BOUNDS_READER(bounds_word_forward)

cudaError_t launch_forward(const void* vol, int dtype, int layout, const Geom& g,
                           const float* Rt, int mode, float* out, cudaStream_t stream) {
    if (dtype == 0) return launch_layout<float>(vol, layout, g, Rt, mode, out, stream);
    return launch_layout<uint16_t>(vol, layout, g, Rt, mode, out, stream);
}

}  // namespace drr

// drr_forward.cu -- forward DRR ray-march kernels (sm_100a).
//
// One thread per ray, a 16 x 16 pixel tile per CTA (warps own 8 x 4
// sub-tiles).  Per ray: view/ray setup and slab clip (drr_internal.cuh),
// then n_samples midpoint samples of the zero-padded trilinear interpolant,
// summed in fp32, then I = density_factor * dt * sum written raw or as
// 1 - exp(-I) (flashdrr.rendering API docs, VolumeRaycaster.__init__:
// ray_samples, density_factor, use_beer_lambert).  Nothing per sample is
// materialised in memory: the fused design the FlashDRR page credits for its
// near-constant footprint ("Memory Scaling").
//
// Two storage layouts, one loop: the caller's linear array, or the array
// inside a one-voxel zero border (drr_prepare_volume).  Sample positions are
// 32.32 fixed point (drr_internal.cuh), clipped per ray so that every corner
// read stays inside the stored volume; inside the voxel-centre box the linear
// layout's upper corner at n-1 is reached with weight 1 - 2^-32 instead of
// through the border, an O(2^-32) difference.
#include <cuda_runtime.h>
#include <stdint.h>

#include "drr_internal.cuh"

namespace drr {
namespace {

template <typename T>
__device__ __forceinline__ float load_voxel(const T* p);

template <>
__device__ __forceinline__ float load_voxel<float>(const float* p) {
    return __ldg(p);
}

// bf16 voxels are stored as their 16-bit patterns; widening to fp32 is exact.
template <>
__device__ __forceinline__ float load_voxel<uint16_t>(const uint16_t* p) {
    return __uint_as_float(((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p))) << 16);
}

template <typename T>
__device__ __forceinline__ float trilinear_at(const T* __restrict__ base, int row, int slice,
                                              float fx, float fy, float fz) {
    const float v000 = load_voxel(base);
    const float v100 = load_voxel(base + 1);
    const float v010 = load_voxel(base + row);
    const float v110 = load_voxel(base + row + 1);
    const float v001 = load_voxel(base + slice);
    const float v101 = load_voxel(base + slice + 1);
    const float v011 = load_voxel(base + slice + row);
    const float v111 = load_voxel(base + slice + row + 1);
    const float c00 = fmaf(fx, v100 - v000, v000);
    const float c10 = fmaf(fx, v110 - v010, v010);
    const float c01 = fmaf(fx, v101 - v001, v001);
    const float c11 = fmaf(fx, v111 - v011, v011);
    const float c0 = fmaf(fy, c10 - c00, c00);
    const float c1 = fmaf(fy, c11 - c01, c01);
    return fmaf(fz, c1 - c0, c0);
}

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
        acc += trilinear_at(vol + idx, row, slice, fix_frac(qx), fix_frac(qy), fix_frac(qz));
        qx += sx;
        qy += sy;
        qz += sz;
    }
    return acc;
}

template <typename T, bool PADDED, int MODE>
__global__ void __launch_bounds__(kThreads)
forward_kernel(const T* __restrict__ vol, const float* __restrict__ Rt, float* __restrict__ out,
               const Geom g) {
    __shared__ View sv;
    const int b = blockIdx.z;
    if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)b, g, sv);
    __syncthreads();
    int r, c;
    tile_pixel(r, c);
    if (r >= g.H || c >= g.W) return;
    Ray ray;
    float result = 0.0f;
    if (ray_setup(sv, g, (double)c, (double)r, PADDED ? 1.0 : 0.0, ray)) {
        const float I = (g.density_factor * ray.dt) * march(vol, g, ray);
        result = (MODE == 1) ? -expm1f(-I) : I;
    }
    out[((size_t)b * g.H + r) * g.W + c] = result;
}

template <typename T, bool PADDED>
cudaError_t launch_typed(const void* vol, const Geom& g, const float* Rt, int mode, float* out,
                         cudaStream_t stream) {
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    const T* v = static_cast<const T*>(vol);
    if (mode == 1)
        forward_kernel<T, PADDED, 1><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    else
        forward_kernel<T, PADDED, 0><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward(const void* vol, int dtype, int layout, const Geom& g,
                           const float* Rt, int mode, float* out, cudaStream_t stream) {
    const bool padded = layout == 1;
    if (dtype == 0)
        return padded ? launch_typed<float, true>(vol, g, Rt, mode, out, stream)
                      : launch_typed<float, false>(vol, g, Rt, mode, out, stream);
    return padded ? launch_typed<uint16_t, true>(vol, g, Rt, mode, out, stream)
                  : launch_typed<uint16_t, false>(vol, g, Rt, mode, out, stream);
}

}  // namespace drr

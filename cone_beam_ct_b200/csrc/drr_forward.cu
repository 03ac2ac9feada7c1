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
// Two storage layouts:
//  * PADDED: the volume sits inside a one-voxel zero border, so the border
//    *is* the zero padding and the loop needs no clamps.  Memory safety comes
//    from a per-ray check: samples are fma(i, S, Q0) and fma rounding is
//    monotone in i, so if the first and the last sample lie inside the padded
//    box, every sample does.
//  * LINEAR: the caller's plain array; each sample is clamped into
//    [0, n-1) per axis before the floor.  Inside the voxel-centre box that is
//    the same interpolant (the upper corner at n-1 gets weight 0 either way);
//    outside it, which only rounding at the box faces can reach, the result
//    differs from zero padding by O(ulp).
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

// Sum of the N samples of one ray in the padded layout.  Returns false if the
// ray's samples would leave the padded box (only possible for non-finite or
// absurd geometry); the caller then treats the ray as a miss.
template <typename T>
__device__ __forceinline__ bool march_padded(const T* __restrict__ vol, const Geom& g,
                                             const Ray& ray, float& sum) {
    float q0[3], ql[3];
    const float last = (float)(g.N - 1);
    const float lim[3] = {(float)(g.nx + 1), (float)(g.ny + 1), (float)(g.nz + 1)};
    bool inside = true;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        q0[k] = fmaf(0.5f, ray.S[k], ray.P[k] + 1.0f);      // padded coordinate of sample 0
        ql[k] = fmaf(last, ray.S[k], q0[k]);                // ... of sample N-1
        inside = inside && q0[k] >= 0.0f && q0[k] < lim[k] && ql[k] >= 0.0f && ql[k] < lim[k];
    }
    if (!inside) return false;
    const int row = g.row, slice = g.slice;
    float acc = 0.0f, fi = 0.0f;
#pragma unroll 4
    for (int i = 0; i < g.N; ++i, fi += 1.0f) {
        const float qx = fmaf(fi, ray.S[0], q0[0]);
        const float qy = fmaf(fi, ray.S[1], q0[1]);
        const float qz = fmaf(fi, ray.S[2], q0[2]);
        int ix, iy, iz;
        const float fx = qx - floor_small(qx, ix);
        const float fy = qy - floor_small(qy, iy);
        const float fz = qz - floor_small(qz, iz);
        const int idx = iz * slice + iy * row + ix;
        acc += trilinear_at(vol + idx, row, slice, fx, fy, fz);
    }
    sum = acc;
    return true;
}

// Sum of the N samples of one ray in the caller's linear layout (clamped).
template <typename T>
__device__ __forceinline__ float march_linear(const T* __restrict__ vol, const Geom& g,
                                              const Ray& ray) {
    float p0[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) p0[k] = fmaf(0.5f, ray.S[k], ray.P[k]);
    const int row = g.row, slice = g.slice;
    const float hx = g.hi_clamp[0], hy = g.hi_clamp[1], hz = g.hi_clamp[2];
    float acc = 0.0f, fi = 0.0f;
#pragma unroll 4
    for (int i = 0; i < g.N; ++i, fi += 1.0f) {
        const float qx = fminf(fmaxf(fmaf(fi, ray.S[0], p0[0]), 0.0f), hx);
        const float qy = fminf(fmaxf(fmaf(fi, ray.S[1], p0[1]), 0.0f), hy);
        const float qz = fminf(fmaxf(fmaf(fi, ray.S[2], p0[2]), 0.0f), hz);
        int ix, iy, iz;
        const float fx = qx - floor_small(qx, ix);
        const float fy = qy - floor_small(qy, iy);
        const float fz = qz - floor_small(qz, iz);
        const int idx = iz * slice + iy * row + ix;
        acc += trilinear_at(vol + idx, row, slice, fx, fy, fz);
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
    if (ray_setup(sv, g, (float)c, (float)r, ray)) {
        float sum = 0.0f;
        bool ok = true;
        if (PADDED)
            ok = march_padded(vol, g, ray, sum);
        else
            sum = march_linear(vol, g, ray);
        if (ok) {
            const float I = (g.density_factor * ray.dt) * sum;
            result = (MODE == 1) ? -expm1f(-I) : I;
        }
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

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
    float hi_clamp[3];       // largest float below n - 1 (linear-layout clamp)
    float inv_sp[3];         // 1 / spacing
    float origin[3];         // world mm of voxel 0's centre
    float kinv[6];           // K^-1 = [k0 k1 k2; 0 k3 k4; 0 0 k5]
    int B, H, W, N;
    float density_factor;
};

// Per-view quantities, computed once per CTA from the view's [R|t]:
//   A = R^T K^-1  (pixel (u, v, 1) -> world direction, unnormalised)
//   C = (-R^T t - origin) / spacing  (camera centre in IJK)
struct View {
    float A[9];
    float C[3];
};

__device__ __forceinline__ void view_setup(const float* __restrict__ Rt12, const Geom& g,
                                           View& v) {
    float R[9], t[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
#pragma unroll
        for (int c = 0; c < 3; ++c) R[3 * r + c] = Rt12[4 * r + c];
        t[r] = Rt12[4 * r + 3];
    }
    const float i00 = g.kinv[0], i01 = g.kinv[1], i02 = g.kinv[2];
    const float i11 = g.kinv[3], i12 = g.kinv[4], i22 = g.kinv[5];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        // column a of R is row a of R^T
        const float r0 = R[a], r1 = R[3 + a], r2 = R[6 + a];
        v.A[3 * a + 0] = r0 * i00;
        v.A[3 * a + 1] = fmaf(r0, i01, r1 * i11);
        v.A[3 * a + 2] = fmaf(r0, i02, fmaf(r1, i12, r2 * i22));
        const float cw = -fmaf(r0, t[0], fmaf(r1, t[1], r2 * t[2]));
        v.C[a] = (cw - g.origin[a]) * g.inv_sp[a];
    }
}

// One ray, clipped and discretised: sample i sits at P + (i + 1/2) * S in
// IJK coordinates; dt is the sample spacing in world mm.
struct Ray {
    float P[3];
    float S[3];
    float dt;
};

// Returns false for a miss (or a ray whose geometry is not finite).
__device__ __forceinline__ bool ray_setup(const View& v, const Geom& g, float u, float w,
                                          Ray& ray) {
    float a[3], d[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) a[k] = fmaf(v.A[3 * k], u, fmaf(v.A[3 * k + 1], w, v.A[3 * k + 2]));
    const float n2 = fmaf(a[0], a[0], fmaf(a[1], a[1], a[2] * a[2]));
    const float rn = 1.0f / sqrtf(n2);
    float t_near = -INFINITY, t_far = INFINITY;
    bool ok = true;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        d[k] = a[k] * rn * g.inv_sp[k];
        const float c = v.C[k];
        ok = ok && isfinite(d[k]) && isfinite(c);
        if (d[k] != 0.0f) {
            const float inv = 1.0f / d[k];
            const float ta = (0.0f - c) * inv;
            const float tb = (g.hi[k] - c) * inv;
            t_near = fmaxf(t_near, fminf(ta, tb));
            t_far = fminf(t_far, fmaxf(ta, tb));
        } else {
            // parallel to this slab: inside (planes included) or a miss
            ok = ok && (c >= 0.0f) && (c <= g.hi[k]);
        }
    }
    const float t0 = fmaxf(t_near, 0.0f);
    const float t1 = t_far;
    if (!ok || !(t1 > t0) || !isfinite(t1)) return false;
    const float dt = (t1 - t0) / (float)g.N;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        ray.P[k] = fmaf(t0, d[k], v.C[k]);
        ray.S[k] = dt * d[k];
    }
    ray.dt = dt;
    return true;
}

// floor(x) for 0 <= x < 2^22 with full-rate FP32 ops only: adding 1.5 * 2^23
// with round-down leaves floor(x) in the low mantissa bits.
__device__ __forceinline__ float floor_small(float x, int& xi) {
    const float kMagic = 12582912.0f;            // 1.5 * 2^23, bit pattern 0x4B400000
    const float t = __fadd_rd(x, kMagic);
    xi = __float_as_int(t) - 0x4B400000;
    return t - kMagic;                           // exact
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
// host-side launchers (defined in the .cu files)

cudaError_t launch_forward(const void* vol, int dtype, int layout, const Geom& g,
                           const float* Rt, int mode, float* out, cudaStream_t stream);
cudaError_t launch_adjoint(const Geom& g, const float* Rt, int mode, const float* grad_out,
                           const float* fwd_out, float* grad_vol, cudaStream_t stream);
cudaError_t launch_prepare(const float* src, int nx, int ny, int nz, int dtype, int layout,
                           void* dst, cudaStream_t stream);

}  // namespace drr

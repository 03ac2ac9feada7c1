// drr_adjoint.cu -- adjoint (volume gradient) of the DRR ray-march (sm_100a).
//
// The transpose of the forward operator (TorchTomo page, "Discrete Adjoint
// and Learned Primal-Dual": <A x, y> = <x, A^T y>): every sample of every
// ray scatters g * w_corner into the 8 voxels its trilinear interpolation
// read, with g = grad_out * density_factor * dt per ray, times exp(-I) =
// 1 - out in Beer-Lambert mode (the derivative of 1 - exp(-I)).  This is the
// backward kernel of the fused renderer (FlashDRR page, "Train vs. Eval
// Dynamics").  Same launch shape, ray setup and 32.32 sample positions as the
// forward on the linear layout, so its weights are the forward's weights and
// the adjoint is that forward's transpose up to fp32 rounding.
#include <cuda_runtime.h>
#include <stdint.h>

#include "drr_internal.cuh"

namespace drr {
namespace {

template <int MODE>
__global__ void __launch_bounds__(kThreads)
adjoint_kernel(const float* __restrict__ Rt, const float* __restrict__ grad_out,
               const float* __restrict__ fwd_out, float* __restrict__ grad, const Geom g) {
    __shared__ View sv;
    const int b = blockIdx.z;
    if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)b, g, sv);
    __syncthreads();
    int r, c;
    tile_pixel(r, c);
    if (r >= g.H || c >= g.W) return;
    const size_t pix = ((size_t)b * g.H + r) * g.W + c;
    float go = grad_out[pix];
    if (MODE == 1) go *= 1.0f - fwd_out[pix];
    Ray ray;
    if (go == 0.0f || !ray_setup(sv, g, (double)c, (double)r, 0.0, ray)) return;
    const float scale = go * (g.density_factor * ray.dt);
    const int row = g.row, slice = g.slice;
    long long qx = ray.q0[0], qy = ray.q0[1], qz = ray.q0[2];
    const long long sx = ray.s[0], sy = ray.s[1], sz = ray.s[2];
#pragma unroll 2
    for (int i = 0; i < g.N; ++i) {
        const float fx = fix_frac(qx), fy = fix_frac(qy), fz = fix_frac(qz);
        float* base = grad + (fix_cell(qz) * slice + fix_cell(qy) * row + fix_cell(qx));
        qx += sx;
        qy += sy;
        qz += sz;
        const float wz1 = scale * fz, wz0 = scale * (1.0f - fz);
        const float w01 = wz0 * fy, w00 = wz0 * (1.0f - fy);
        const float w11 = wz1 * fy, w10 = wz1 * (1.0f - fy);
        const float gx = 1.0f - fx;
        atomicAdd(base, w00 * gx);
        atomicAdd(base + 1, w00 * fx);
        atomicAdd(base + row, w01 * gx);
        atomicAdd(base + row + 1, w01 * fx);
        atomicAdd(base + slice, w10 * gx);
        atomicAdd(base + slice + 1, w10 * fx);
        atomicAdd(base + slice + row, w11 * gx);
        atomicAdd(base + slice + row + 1, w11 * fx);
    }
}

}  // namespace

cudaError_t launch_adjoint(const Geom& g, const float* Rt, int mode, const float* grad_out,
                           const float* fwd_out, float* grad_vol, cudaStream_t stream) {
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    if (mode == 1)
        adjoint_kernel<1><<<grid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, grad_vol, g);
    else
        adjoint_kernel<0><<<grid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, grad_vol, g);
    return cudaGetLastError();
}

}  // namespace drr

// drr_adjoint.cu -- adjoint (volume gradient) of the DRR ray-march (sm_100a).
//
// The transpose of the forward operator (TorchTomo page, "Discrete Adjoint
// and Learned Primal-Dual": <A x, y> = <x, A^T y>): every sample of every
// ray scatters g * w_corner into the 8 voxels its trilinear interpolation
// read, with g = grad_out * density_factor * dt per ray, times exp(-I) =
// 1 - out in Beer-Lambert mode (the derivative of 1 - exp(-I)).  This is the
// backward kernel of the fused renderer (FlashDRR page, "Train vs. Eval
// Dynamics").  Same ray setup and 32.32 sample positions as the forward on
// the linear layout, so its weights are the forward's weights and the
// adjoint is that forward's transpose up to fp32 rounding.
//
// Where the time goes: the fp32 atomic adds, which the L2 executes at a fixed
// rate of sector operations, and which stall on hot spots when many rays
// cross the same voxels at once.  Three measures cut both:
//  * A pending block per ray: the 8 corner sums of the current cell stay in
//    registers while consecutive samples fall into overlapping cells; when
//    the cell moves by one along an axis only the face that leaves is
//    flushed (4 atomics) and the rest slides over.  Per sample the ray then
//    issues ~4 (|S_x| + |S_y| + |S_z|) atomics instead of 8 (S: the step in
//    voxels), the fewer the denser the sampling.
//  * Phases: each warp of the grid starts its rays at a different eighth of
//    their length (wrapping round), so that warps working on neighbouring
//    rays at the same time are at different depths rather than on the same
//    voxels.
//  * Lane mapping by density: where a 16 x 16 pixel tile spans fewer than 8
//    voxels (rays much closer than a voxel), lanes are spread over the whole
//    tile so that the lanes of one atomic instruction hit different words;
//    otherwise a warp keeps an 8 x 4 block of neighbouring rays, whose
//    atomics share sectors.
// Measured alternatives (shared-memory windows flushed with coalesced global
// atomics; no pending block; no phases) were slower on every workload.
#include <cuda_runtime.h>
#include <stdint.h>

#include "drr_internal.cuh"

namespace drr {
namespace {

// 8 corner sums of a pending block at cell (x, y, z); a[k] belongs to corner
// (k & 1, (k >> 1) & 1, k >> 2).
__device__ __forceinline__ void flush_block(float* __restrict__ grad, const int st[3],
                                            const int cell[3], const float a[8]) {
    float* p = grad + (cell[2] * st[2] + cell[1] * st[1] + cell[0]);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        atomicAdd(p + ((k & 1) ? 1 : 0) + ((k & 2) ? st[1] : 0) + ((k & 4) ? st[2] : 0), a[k]);
}

// Move the pending block one cell along axis AX (d = +1 or -1): flush the face
// that leaves, slide the other face over, start the new face at zero.
template <int AX>
__device__ __forceinline__ void slide(int d, float* __restrict__ grad, const int st[3], int cell[3],
                                      float a[8]) {
    if (d == 0) return;
    const int side = d > 0 ? 0 : 1;                           // face that leaves
    constexpr int A = AX == 0 ? 1 : 0, B = AX == 2 ? 1 : 2;   // the other two axes, ascending
    float* p = grad + (cell[2] * st[2] + cell[1] * st[1] + cell[0]) + (side ? st[AX] : 0);
    float v[4];
    int n = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (((k >> AX) & 1) == 0) v[n++] = side ? a[k | (1 << AX)] : a[k];
    atomicAdd(p, v[0]);
    atomicAdd(p + st[A], v[1]);
    atomicAdd(p + st[B], v[2]);
    atomicAdd(p + st[A] + st[B], v[3]);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (((k >> AX) & 1) != 0) continue;
        const int hi = k | (1 << AX);
        if (d > 0) {
            a[k] = a[hi];
            a[hi] = 0.0f;
        } else {
            a[hi] = a[k];
            a[k] = 0.0f;
        }
    }
    cell[AX] += d;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads)
adjoint_kernel(const float* __restrict__ Rt, const float* __restrict__ grad_out,
               const float* __restrict__ fwd_out, float* __restrict__ grad, const Geom g) {
    __shared__ View sv;
    __shared__ int s_dense;
    const int b = blockIdx.z;
    const int tid = threadIdx.x;
    if (tid == 0) {
        view_setup(Rt + 12 * (size_t)b, g, sv);
        // tile width in voxels where its rays cross the volume centre
        const double u0 = blockIdx.x * kTileW, v0 = blockIdx.y * kTileH;
        double c2 = 0.0, n0 = 0.0, n1 = 0.0, dot = 0.0;
        for (int k = 0; k < 3; ++k) {
            const double d0 = sv.A[3 * k] * u0 + sv.A[3 * k + 1] * v0 + sv.A[3 * k + 2];
            const double d1 = d0 + sv.A[3 * k] * (double)kTileW;
            const double off = (sv.C[k] - 0.5 * g.hi[k]) * g.spacing[k];   // camera to centre, mm
            c2 += off * off;
            n0 += d0 * d0;
            n1 += d1 * d1;
            dot += d0 * d1;
        }
        const double ang = acos(fmin(1.0, fmax(-1.0, dot / sqrt(n0 * n1))));
        const double min_sp = fmin(g.spacing[0], fmin(g.spacing[1], g.spacing[2]));
        s_dense = (sqrt(c2) * ang / min_sp) < 8.0 ? 1 : 0;   // NaN geometry: not dense
    }
    __syncthreads();

    int r, c;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (s_dense) {
        // spread: the 32 lanes of a warp cover the whole 16 x 16 tile (bijective)
        c = blockIdx.x * kTileW + (lane & 7) * 2 + (warp & 1);
        r = blockIdx.y * kTileH + (lane >> 3) * 4 + (warp >> 1);
    } else {
        tile_pixel(r, c);
    }
    if (r >= g.H || c >= g.W) return;
    const size_t pix = ((size_t)b * g.H + r) * g.W + c;
    float go = grad_out[pix];
    if (MODE == 1) go *= 1.0f - fwd_out[pix];
    Ray ray;
    if (go == 0.0f || !ray_setup(sv, g, (double)c, (double)r, 0.0, ray)) return;
    const float scale = go * (g.density_factor * ray.dt);
    const int st[3] = {1, g.row, g.slice};

    // phase: this warp starts at sample `start` and wraps round to 0
    const int ph = (warp + blockIdx.x * 3 + blockIdx.y * 5 + blockIdx.z) & 7;
    const int start = (int)(((long long)g.N * ph) >> 3);
    int cell[3];
    float a[8];
    for (int pass = 0; pass < 2; ++pass) {
        const int i0 = pass == 0 ? start : 0;
        const int i1 = pass == 0 ? g.N : start;
        if (i0 >= i1) continue;
        long long qx = ray.q0[0] + (long long)i0 * ray.s[0];
        long long qy = ray.q0[1] + (long long)i0 * ray.s[1];
        long long qz = ray.q0[2] + (long long)i0 * ray.s[2];
        cell[0] = fix_cell(qx);
        cell[1] = fix_cell(qy);
        cell[2] = fix_cell(qz);
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = 0.0f;
        for (int i = i0; i < i1; ++i) {
            const int cx = fix_cell(qx), cy = fix_cell(qy), cz = fix_cell(qz);
            const int dx = cx - cell[0], dy = cy - cell[1], dz = cz - cell[2];
            if (dx < -1 || dx > 1 || dy < -1 || dy > 1 || dz < -1 || dz > 1) {
                // a step of more than one cell: flush the whole block and restart
                flush_block(grad, st, cell, a);
#pragma unroll
                for (int k = 0; k < 8; ++k) a[k] = 0.0f;
                cell[0] = cx;
                cell[1] = cy;
                cell[2] = cz;
            } else {
                slide<0>(dx, grad, st, cell, a);
                slide<1>(dy, grad, st, cell, a);
                slide<2>(dz, grad, st, cell, a);
            }
            const float fx = fix_frac(qx), fy = fix_frac(qy), fz = fix_frac(qz);
            const float wz1 = scale * fz, wz0 = scale * (1.0f - fz);
            const float w00 = wz0 * (1.0f - fy), w01 = wz0 * fy;
            const float w10 = wz1 * (1.0f - fy), w11 = wz1 * fy;
            const float gx = 1.0f - fx;
            a[0] += w00 * gx;
            a[1] += w00 * fx;
            a[2] += w01 * gx;
            a[3] += w01 * fx;
            a[4] += w10 * gx;
            a[5] += w10 * fx;
            a[6] += w11 * gx;
            a[7] += w11 * fx;
            qx += ray.s[0];
            qy += ray.s[1];
            qz += ray.s[2];
        }
        flush_block(grad, st, cell, a);
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

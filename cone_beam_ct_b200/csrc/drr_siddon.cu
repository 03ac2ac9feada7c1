// drr_siddon.cu -- the cell-constant (Siddon) projector and its exact
// adjoint (sm_100a).
//
// The second discretisation of the line integral (diffct page, Features:
// project() and backproject() form an exact adjoint pair for the
// cell-constant Siddon model): voxel (i, j, k) is the cube of side one voxel
// centred on (i, j, k) in IJK with the constant value vol[k][j][i]; a ray's
// image is density_factor times the exact integral of that piecewise-constant
// function along the ray, clipped to the cells' box [-1/2, n - 1/2] per axis
// (t0 = max(t_near, 0)), written raw or as 1 - exp(-I).
//
// One thread per ray walks the cells the ray crosses in order (a 3-D DDA):
// the parameters of the next plane x_a = c_a +- 1/2 on each axis are kept in
// fp64 (advanced by exact multiples of 1/|d_a|, so 256-cell walks keep
// ~1e-13 mm of error), each piece's length goes to the current cell, and
// the axis whose plane comes first advances.  The walk ends at t1 or when a
// cell index leaves the volume, and takes at most nx + ny + nz + 2 steps.
// The backprojection walks the same cells and adds scale * length to each
// with an fp32 atomic (the transpose, term by term).
#include <cuda_runtime.h>
#include <stdint.h>

#include "drr_internal.cuh"

namespace drr {
namespace {

template <typename T>
__device__ __forceinline__ float voxel_value(const T* p);
template <>
__device__ __forceinline__ float voxel_value<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float voxel_value<uint16_t>(const uint16_t* p) {
    return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p)) << 16);
}

// The walk's state for one ray.  Indexed only by constants (walk_step picks
// the axis with selects), so it lives in registers: indexing it by the axis
// number put it in local memory (a 96-byte stack frame; B200, 256^3 fp32
// volume, 4 views of 1024^2: forward 7.18 -> 4.61 ms, backprojection 15.26
// -> 7.09 ms).
struct Walk {
    double t, t1;          // current parameter (mm) and the exit
    double next[3];        // parameter of the next plane on each axis (inf: parallel)
    double delta[3];       // 1 / |d_a|: parameter between planes
    int cell[3], step[3];  // current cell, +-1 per axis
    int didx[3];           // change of the linear index for a step along each axis
    int idx;               // linear index of the cell
};

// Clip to the cells' box and set up the walk; false on a miss.
__device__ __forceinline__ bool walk_setup(const View& v, const Geom& g, double u, double w,
                                           Walk& k) {
    double a[3], d[3];
#pragma unroll
    for (int q = 0; q < 3; ++q) a[q] = v.A[3 * q] * u + v.A[3 * q + 1] * w + v.A[3 * q + 2];
    const double rn = 1.0 / sqrt(a[0] * a[0] + a[1] * a[1] + a[2] * a[2]);
    const int n[3] = {g.nx, g.ny, g.nz};
    double t_near = -INFINITY, t_far = INFINITY;
    bool ok = true;
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        d[q] = a[q] * rn / g.spacing[q];
        const double c = v.C[q], lo = -0.5, hi = (double)n[q] - 0.5;
        ok = ok && isfinite(d[q]) && isfinite(c);
        if (d[q] != 0.0) {
            const double ta = (lo - c) / d[q], tb = (hi - c) / d[q];
            t_near = fmax(t_near, fmin(ta, tb));
            t_far = fmin(t_far, fmax(ta, tb));
        } else {
            ok = ok && c >= lo && c <= hi;
        }
    }
    const double t0 = fmax(t_near, 0.0);
    if (!ok || !(t_far > t0) || !isfinite(t_far)) return false;
    k.t = t0;
    k.t1 = t_far;
    // the first cell: the one holding a point just inside the entry (its
    // midpoint with the next plane would do as well; the cell at the entry
    // point itself may round to either side of a face)
    const double tin = t0 + 1e-9 * fmax(1.0, t_far - t0);
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        const double p = v.C[q] + fmin(tin, 0.5 * (t0 + t_far)) * d[q];
        int c = (int)floor(p + 0.5);
        c = min(max(c, 0), n[q] - 1);
        k.cell[q] = c;
        if (d[q] > 0.0) {
            k.step[q] = 1;
            k.delta[q] = 1.0 / d[q];
            k.next[q] = ((double)c + 0.5 - v.C[q]) / d[q];
        } else if (d[q] < 0.0) {
            k.step[q] = -1;
            k.delta[q] = -1.0 / d[q];
            k.next[q] = ((double)c - 0.5 - v.C[q]) / d[q];
        } else {
            k.step[q] = 0;
            k.delta[q] = INFINITY;
            k.next[q] = INFINITY;
        }
    }
    k.idx = (k.cell[2] * g.ny + k.cell[1]) * g.nx + k.cell[0];
    k.didx[0] = k.step[0];
    k.didx[1] = k.step[1] * g.nx;
    k.didx[2] = k.step[2] * g.nx * g.ny;
    return true;
}

// One step: the length of the current piece; advances to the next cell.
// Returns false when the walk has left the box (the piece is still valid).
__device__ __forceinline__ bool walk_step(const Geom& g, Walk& k, double& len) {
    // the axis whose plane comes first (ties: the lower axis)
    const bool y_first = k.next[1] < k.next[0];
    const double t01 = y_first ? k.next[1] : k.next[0];
    const bool a2 = k.next[2] < t01;
    const double tn = a2 ? k.next[2] : t01;
    const bool a1 = y_first && !a2, a0 = !y_first && !a2;
    const double te = fmin(tn, k.t1);
    len = fmax(te - k.t, 0.0);
    k.t = fmax(k.t, te);
    if (tn >= k.t1) return false;
    if (a0) {
        k.cell[0] += k.step[0];
        k.next[0] += k.delta[0];
    }
    if (a1) {
        k.cell[1] += k.step[1];
        k.next[1] += k.delta[1];
    }
    if (a2) {
        k.cell[2] += k.step[2];
        k.next[2] += k.delta[2];
    }
    const int c = a0 ? k.cell[0] : (a1 ? k.cell[1] : k.cell[2]);
    const int n = a0 ? g.nx : (a1 ? g.ny : g.nz);
    if (c < 0 || c >= n) return false;
    k.idx += a0 ? k.didx[0] : (a1 ? k.didx[1] : k.didx[2]);
    return true;
}

template <typename T, int MODE>
__global__ void __launch_bounds__(kThreads)
siddon_forward_kernel(const T* __restrict__ vol, const float* __restrict__ Rt,
                      float* __restrict__ out, const Geom g) {
    __shared__ View sv;
    const int b = blockIdx.z;
    if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)b, g, sv);
    __syncthreads();
    int r, c;
    tile_pixel(r, c);
    if (r >= g.H || c >= g.W) return;
    float result = 0.0f;
    Walk k;
    if (walk_setup(sv, g, (double)c, (double)r, k)) {
        float acc = 0.0f;
        const int max_steps = g.nx + g.ny + g.nz + 2;
        for (int s = 0; s < max_steps; ++s) {
            const int idx = k.idx;               // in the volume: checked before every step
            double len;
            const bool more = walk_step(g, k, len);
            if (in_bounds(idx, 1, (long long)g.nx * g.ny * g.nz))
                acc = fmaf((float)len, voxel_value(vol + idx), acc);
            if (!more) break;
        }
        const float I = g.density_factor * acc;
        result = MODE == 1 ? -expm1f(-I) : I;
    }
    const long long pix = ((long long)b * g.H + r) * g.W + c;
    if (in_bounds(pix, 1, (long long)g.B * g.H * g.W)) out[pix] = result;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads)
siddon_adjoint_kernel(const float* __restrict__ Rt, const float* __restrict__ grad_out,
                      const float* __restrict__ fwd_out, float* __restrict__ grad, const Geom g) {
    __shared__ View sv;
    const int b = blockIdx.z;
    if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)b, g, sv);
    __syncthreads();
    int r, c;
    tile_pixel(r, c);
    if (r >= g.H || c >= g.W) return;
    const size_t pix = ((size_t)b * g.H + r) * g.W + c;
    if (!in_bounds(pix, 1, (long long)g.B * g.H * g.W)) return;
    float go = grad_out[pix];
    if (MODE == 1) go *= 1.0f - fwd_out[pix];
    Walk k;
    if (go == 0.0f || !walk_setup(sv, g, (double)c, (double)r, k)) return;
    const float scale = go * g.density_factor;
    const int max_steps = g.nx + g.ny + g.nz + 2;
    for (int s = 0; s < max_steps; ++s) {
        const int idx = k.idx;
        double len;
        const bool more = walk_step(g, k, len);
        if (len > 0.0 && in_bounds(idx, 1, (long long)g.nx * g.ny * g.nz))
            atomicAdd(grad + idx, scale * (float)len);
        if (!more) break;
    }
}

}  // namespace

DRR_BOUNDS_READER(bounds_word_siddon)

cudaError_t launch_siddon(const void* vol, int dtype, const Geom& g, const float* Rt, int mode,
                          float* out, cudaStream_t stream) {
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    if (dtype == 0) {
        const float* v = static_cast<const float*>(vol);
        if (mode == 1) siddon_forward_kernel<float, 1><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
        else siddon_forward_kernel<float, 0><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    } else {
        const uint16_t* v = static_cast<const uint16_t*>(vol);
        if (mode == 1) siddon_forward_kernel<uint16_t, 1><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
        else siddon_forward_kernel<uint16_t, 0><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    }
    return cudaGetLastError();
}

cudaError_t launch_siddon_adjoint(const Geom& g, const float* Rt, int mode, const float* grad_out,
                                  const float* fwd_out, float* grad_vol, cudaStream_t stream) {
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    if (mode == 1)
        siddon_adjoint_kernel<1><<<grid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, grad_vol, g);
    else
        siddon_adjoint_kernel<0><<<grid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, grad_vol, g);
    return cudaGetLastError();
}

}  // namespace drr

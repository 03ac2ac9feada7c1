// drr_prepare.cu -- volume re-layout / conversion kernels (sm_100a).
//
// fp32 -> bf16 storage rounds to nearest even (the bf16 rendering mode of
// nanodrr's page, "Benchmarks": mixed precision; here storage only, the
// arithmetic stays fp32).  The padded layout surrounds the volume with a
// one-voxel zero border, which is exactly the zero padding of the trilinear
// interpolation.  The corner-replicated layout stores every cell's 8 corner
// voxels together.  Plain grid-stride loops: a one-off HBM-bound copy.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "drr_internal.cuh"

namespace drr {
namespace {

template <typename T>
__device__ __forceinline__ T store_value(float x);

template <>
__device__ __forceinline__ float store_value<float>(float x) {
    return x;
}

template <>
__device__ __forceinline__ uint16_t store_value<uint16_t>(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

template <typename T>
__global__ void to_linear(const float* __restrict__ src, T* __restrict__ dst, int64_t n) {
    for (int64_t m = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; m < n;
         m += (int64_t)gridDim.x * blockDim.x)
        dst[m] = store_value<T>(__ldg(src + m));
}

template <typename T>
__global__ void to_padded(const float* __restrict__ src, T* __restrict__ dst, int nx, int ny,
                          int nz) {
    const int px = nx + 2, py = ny + 2;
    const int64_t n = (int64_t)px * py * (nz + 2);
    for (int64_t m = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; m < n;
         m += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(m % px);
        const int j = (int)((m / px) % py);
        const int k = (int)(m / ((int64_t)px * py));
        float v = 0.0f;
        const int64_t at = ((int64_t)(k - 1) * ny + (j - 1)) * nx + (i - 1);
        if (i >= 1 && i <= nx && j >= 1 && j <= ny && k >= 1 && k <= nz &&
            in_bounds(at, 1, (int64_t)nx * ny * nz))
            v = __ldg(src + at);
        dst[m] = store_value<T>(v);
    }
}

// Corner-replicated layout: record m = cell (i, j, k) holds the 8 voxels
// src[k+c][j+b][i+a] in the order a + 2b + 4c, written as one (bf16) or two
// (fp32) 16-byte stores.
__device__ __forceinline__ void store_corners(float* dst, const float v[8]) {
    float4* d = reinterpret_cast<float4*>(dst);
    d[0] = make_float4(v[0], v[1], v[2], v[3]);
    d[1] = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ void store_corners(uint16_t* dst, const float v[8]) {
    unsigned w[4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
        w[m] = (unsigned)store_value<uint16_t>(v[2 * m]) |
               ((unsigned)store_value<uint16_t>(v[2 * m + 1]) << 16);
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// A CTA takes whole x rows of cells (one 32-bit division per row for j and
// k, not 64-bit divisions per record), its threads consecutive cells of the
// row: coalesced stores.  B200, 256^3: bf16 corner records 0.102 -> 0.082
// ms, fp32 quads 0.097 -> 0.072 ms.
template <typename T>
__global__ void to_corners(const float* __restrict__ src, T* __restrict__ dst, int nx, int ny,
                           int nz) {
    const int cx = nx - 1, cy = ny - 1;
    const int rows = cy * (nz - 1);              // < 2^31: stored elements are capped
    const int64_t sy = nx, sz = (int64_t)nx * ny;
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        const int k = row / cy, j = row - k * cy;
        const int64_t base = ((int64_t)k * ny + j) * nx;
        for (int i = threadIdx.x; i < cx; i += blockDim.x) {
            const int64_t at = base + i, m = (int64_t)row * cx + i;
            const float* p = src + at;
            // corner (a, b, c) at element a + 2b + 4c
            float v[8];
            const bool ok = in_bounds(at, sz + sy + 2, sz * nz);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                v[e] = ok ? __ldg(p + ((e & 1) ? 1 : 0) + ((e & 2) ? sy : 0) + ((e & 4) ? sz : 0))
                          : 0.0f;
            store_corners(dst + m * 8, v);
        }
    }
}

// xy-quad layout: quad m = (i, j, k) holds src[k][j+b][i+a] in the order
// a + 2b, one 16-byte (fp32) or 8-byte (bf16) store.
template <typename T>
__global__ void to_quads(const float* __restrict__ src, T* __restrict__ dst, int nx, int ny,
                         int nz) {
    const int qx = nx - 1, qy = ny - 1;
    const int rows = qy * nz;                    // whole x rows per CTA, as to_corners
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        const int k = row / qy, j = row - k * qy;
        const int64_t base = ((int64_t)k * ny + j) * nx;
        for (int i = threadIdx.x; i < qx; i += blockDim.x) {
            const int64_t at = base + i, m = (int64_t)row * qx + i;
            const float* p = src + at;
            const bool ok = in_bounds(at, (int64_t)nx + 2, (int64_t)nx * ny * nz);
            const float v[4] = {ok ? __ldg(p) : 0.0f, ok ? __ldg(p + 1) : 0.0f,
                                ok ? __ldg(p + nx) : 0.0f, ok ? __ldg(p + nx + 1) : 0.0f};
            if constexpr (sizeof(T) == 4) {
                reinterpret_cast<float4*>(dst)[m] = make_float4(v[0], v[1], v[2], v[3]);
            } else {
                const unsigned w0 = (unsigned)store_value<uint16_t>(v[0]) |
                                    ((unsigned)store_value<uint16_t>(v[1]) << 16);
                const unsigned w1 = (unsigned)store_value<uint16_t>(v[2]) |
                                    ((unsigned)store_value<uint16_t>(v[3]) << 16);
                reinterpret_cast<uint2*>(dst)[m] = make_uint2(w0, w1);
            }
        }
    }
}

// CTAs for a pass over `rows` rows, one row per CTA at a time: every SM
// filled, the loops stride over the rest.
int rows_grid(int64_t rows) {
    const int64_t cap = 148 * 8;
    return (int)(rows < cap ? (rows > 0 ? rows : 1) : cap);
}

int grid_for(int64_t n) {
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = 148 * 16;   // enough CTAs to fill every SM; the loops stride
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

// Bricked layout: element m of the output is element m % kBrickStride of
// brick m / kBrickStride; a brick's elements past its (kBrick + 1)^3 voxels,
// and voxels past the volume's edge, are zero.
template <typename T>
__global__ void to_bricks(const float* __restrict__ src, T* __restrict__ dst, int nx, int ny,
                          int nz) {
    const int nbx = brick_count(nx), nby = brick_count(ny);
    const int64_t n = (int64_t)nbx * nby * brick_count(nz) * kBrickStride;
    for (int64_t m = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; m < n;
         m += (int64_t)gridDim.x * blockDim.x) {
        const int64_t brick = m / kBrickStride;
        const int e = (int)(m - brick * kBrickStride);
        float v = 0.0f;
        if (e < kBrickPlane * kBrickEdge) {
            const int lz = e / kBrickPlane, ly = (e / kBrickEdge) % kBrickEdge, lx = e % kBrickEdge;
            const int bx = (int)(brick % nbx), by = (int)((brick / nbx) % nby);
            const int bz = (int)(brick / ((int64_t)nbx * nby));
            const int i = bx * kBrick + lx, j = by * kBrick + ly, k = bz * kBrick + lz;
            const int64_t at = ((int64_t)k * ny + j) * nx + i;
            if (i < nx && j < ny && k < nz && in_bounds(at, 1, (int64_t)nx * ny * nz))
                v = __ldg(src + at);
        }
        dst[m] = store_value<T>(v);
    }
}

}  // namespace

DRR_BOUNDS_READER(bounds_word_prepare)

cudaError_t launch_prepare(const float* src, int nx, int ny, int nz, int dtype, int layout,
                           void* dst, cudaStream_t stream) {
    if (layout == 0) {
        const int64_t n = (int64_t)nx * ny * nz;
        if (dtype == 0)
            to_linear<float><<<grid_for(n), 256, 0, stream>>>(src, static_cast<float*>(dst), n);
        else
            to_linear<uint16_t><<<grid_for(n), 256, 0, stream>>>(src, static_cast<uint16_t*>(dst),
                                                                 n);
    } else if (layout == 4) {
        const int64_t n =
            (int64_t)brick_count(nx) * brick_count(ny) * brick_count(nz) * kBrickStride;
        if (dtype == 0)
            to_bricks<float><<<grid_for(n), 256, 0, stream>>>(src, static_cast<float*>(dst), nx,
                                                              ny, nz);
        else
            to_bricks<uint16_t><<<grid_for(n), 256, 0, stream>>>(src, static_cast<uint16_t*>(dst),
                                                                 nx, ny, nz);
    } else if (layout == 3) {
        const int64_t n = (int64_t)(ny - 1) * nz;       // rows of quads
        if (dtype == 0)
            to_quads<float><<<rows_grid(n), 256, 0, stream>>>(src, static_cast<float*>(dst), nx,
                                                              ny, nz);
        else
            to_quads<uint16_t><<<rows_grid(n), 256, 0, stream>>>(src, static_cast<uint16_t*>(dst),
                                                                nx, ny, nz);
    } else if (layout == 2) {
        const int64_t n = (int64_t)(ny - 1) * (nz - 1);  // rows of cells
        if (dtype == 0)
            to_corners<float><<<rows_grid(n), 256, 0, stream>>>(src, static_cast<float*>(dst), nx,
                                                               ny, nz);
        else
            to_corners<uint16_t><<<rows_grid(n), 256, 0, stream>>>(
                src, static_cast<uint16_t*>(dst), nx, ny, nz);
    } else {
        const int64_t n = (int64_t)(nx + 2) * (ny + 2) * (nz + 2);
        if (dtype == 0)
            to_padded<float><<<grid_for(n), 256, 0, stream>>>(src, static_cast<float*>(dst), nx,
                                                              ny, nz);
        else
            to_padded<uint16_t><<<grid_for(n), 256, 0, stream>>>(
                src, static_cast<uint16_t*>(dst), nx, ny, nz);
    }
    return cudaGetLastError();
}

}  // namespace drr

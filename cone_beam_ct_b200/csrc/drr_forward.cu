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

// One sample in the corner-replicated layout.  A cell record holds corner
// (a, b, c) -- voxel (i + a, j + b, k + c) -- at element a + 2b + 4c.
//
// fp32 records: two 16-byte loads (the corners with c = 0, then c = 1) and
// scalar lerps.  This path is bound by memory latency; a record order with
// a as the slowest index (which lets packed lerps start without moves) ran
// slower here (B200, 512^3 fp32 volume: 5.1 against 4.0 ms; 256^3: 3.07
// against 2.96 ms).
__device__ __forceinline__ float sample_corners(const float* __restrict__ p, float fx, float fy,
                                                float fz) {
    const float4 lo = __ldg(reinterpret_cast<const float4*>(p));       // c = 0: 000 100 010 110
    const float4 hi = __ldg(reinterpret_cast<const float4*>(p) + 1);   // c = 1
    const float c00 = fmaf(fx, lo.y - lo.x, lo.x);
    const float c10 = fmaf(fx, lo.w - lo.z, lo.z);
    const float c01 = fmaf(fx, hi.y - hi.x, hi.x);
    const float c11 = fmaf(fx, hi.w - hi.z, hi.z);
    const float c0 = fmaf(fy, c10 - c00, c00);
    const float c1 = fmaf(fy, c11 - c01, c01);
    return fmaf(fz, c1 - c0, c0);
}

// bf16 records: one 16-byte load, element 2m in the low half of word m, so
// word m holds the x pair (a = 0, 1) of corner row m = b + 2c.  Widening a
// bf16 to fp32 is exact (its bits in the high half): the a = 0 corners are
// widened with a shift; the x differences take the a = 1 corners as bf16
// operands of sm_100's mixed-precision subtraction (sub.f32.bf16 widens its
// bf16 operand exactly and rounds the difference once: the fp32
// subtraction's result).  The 7 lerps then run as 3 packed fp32x2 steps
// (sm_100's FFMA2, one instruction for two lanes of fp32 work) on the row
// pairs (c = 0, c = 1) at b = 0 and b = 1, and one scalar step.  Each lane
// computes exactly what trilinear_at computes (b - a as fma(a, -1, b), which
// rounds once like the subtraction), so the corner layout gives the linear
// layout's bits.
__device__ __forceinline__ float sub_bf16_f32(unsigned short a, float c) {
    float d;
    asm("sub.rn.f32.bf16 %0, %1, %2;" : "=f"(d) : "h"(a), "f"(c));
    return d;
}

__device__ __forceinline__ float sample_corners(const uint16_t* __restrict__ p, float fx, float fy,
                                                float fz) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
    // a = 0 corners of rows (b, c) = (0, 0), (0, 1) and (1, 0), (1, 1),
    // widened by a byte permute (low half to high, zeros below) that runs on
    // the integer pipe rather than the FMA pipe a shift may be issued to
    const float2 lo0 = make_float2(__uint_as_float(__byte_perm(w.x, 0u, 0x1044)),
                                   __uint_as_float(__byte_perm(w.z, 0u, 0x1044)));
    const float2 lo1 = make_float2(__uint_as_float(__byte_perm(w.y, 0u, 0x1044)),
                                   __uint_as_float(__byte_perm(w.w, 0u, 0x1044)));
    const float2 d0 = make_float2(sub_bf16_f32((unsigned short)(w.x >> 16), lo0.x),
                                  sub_bf16_f32((unsigned short)(w.z >> 16), lo0.y));
    const float2 d1 = make_float2(sub_bf16_f32((unsigned short)(w.y >> 16), lo1.x),
                                  sub_bf16_f32((unsigned short)(w.w >> 16), lo1.y));
    const float2 f2 = make_float2(fx, fx);
    const float2 x0 = __ffma2_rn(f2, d0, lo0);                 // (c00, c01): b = 0, c = 0 / 1
    const float2 x1 = __ffma2_rn(f2, d1, lo1);                 // (c10, c11): b = 1
    const float2 m1 = make_float2(-1.0f, -1.0f);
    const float2 y = __ffma2_rn(make_float2(fy, fy), __ffma2_rn(x0, m1, x1), x0);   // (c0, c1)
    return fmaf(fz, y.y - y.x, y.x);
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
        acc += sample_corners(vol + (size_t)cell * 8, fix_frac(qx), fix_frac(qy), fix_frac(qz));
        qx += sx;
        qy += sy;
        qz += sz;
    }
    return acc;
}

template <typename T, int LAYOUT, int MODE>
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
    if (ray_setup(sv, g, (double)c, (double)r, LAYOUT == 1 ? 1.0 : 0.0, ray)) {
        const float sum = LAYOUT == 2 ? march_corners(vol, g, ray) : march(vol, g, ray);
        const float I = (g.density_factor * ray.dt) * sum;
        result = (MODE == 1) ? -expm1f(-I) : I;
    }
    out[((size_t)b * g.H + r) * g.W + c] = result;
}

template <typename T, int LAYOUT>
cudaError_t launch_typed(const void* vol, const Geom& g, const float* Rt, int mode, float* out,
                         cudaStream_t stream) {
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    const T* v = static_cast<const T*>(vol);
    if (mode == 1)
        forward_kernel<T, LAYOUT, 1><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    else
        forward_kernel<T, LAYOUT, 0><<<grid, kThreads, 0, stream>>>(v, Rt, out, g);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_layout(const void* vol, int layout, const Geom& g, const float* Rt, int mode,
                          float* out, cudaStream_t stream) {
    if (layout == 2) return launch_typed<T, 2>(vol, g, Rt, mode, out, stream);
    if (layout == 1) return launch_typed<T, 1>(vol, g, Rt, mode, out, stream);
    return launch_typed<T, 0>(vol, g, Rt, mode, out, stream);
}

}  // namespace

cudaError_t launch_forward(const void* vol, int dtype, int layout, const Geom& g,
                           const float* Rt, int mode, float* out, cudaStream_t stream) {
    if (dtype == 0) return launch_layout<float>(vol, layout, g, Rt, mode, out, stream);
    return launch_layout<uint16_t>(vol, layout, g, Rt, mode, out, stream);
}

}  // namespace drr

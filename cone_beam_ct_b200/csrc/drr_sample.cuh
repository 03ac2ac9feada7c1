// drr_sample.cuh -- one trilinear sample from each stored volume layout
// (include/drr.h), shared by the forward and the alpha-mode adjoint so that
// both read bit-identical sample values.
//
// Zero-padded trilinear interpolation (the grid_sample path of flashdrr's
// VolumeRaycaster): 8 corner voxels, 7 lerps a + f (b - a), x first, then y,
// then z.  Every layout evaluates the same lerps in the same order, so the
// layouts give the same bits.
#pragma once

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

// A voxel read with an ordinary load, from any state space (__ldg is a
// global-memory load: a shared-memory address is not valid for it).
__device__ __forceinline__ float load_voxel_any(const float* p) { return *p; }
__device__ __forceinline__ float load_voxel_any(const uint16_t* p) {
    return __uint_as_float(((uint32_t)*p) << 16);
}

// GLOBAL: the volume is in global memory (read through the read-only path);
// else anywhere, shared memory included.  The same lerps either way.
// Opacity of a sample, a = 1 - exp(-x), x = s mu (front-to-back alpha
// compositing).  fp32 volumes: -expm1f(-x), which keeps its relative
// accuracy for the thin samples of fine sampling.  bf16 volumes: the
// Maclaurin series of 1 - e^-x, x (1 - x/2 (1 - x/3 (1 - x/4 (1 - x/5)))),
// for |x| < 1/8, where the first omitted term, x^6 / 6!, is below 5e-8 of
// the result, and 1 - __expf(-x) above, where the result is at least 0.1175
// and __expf's error stays near fp32 rounding.  Measured on B200 (256^3
// bf16 corner records, 4 views of 1024^2 x 512) against expm1f: alpha
// forward 4.76 -> 4.02 ms, its pose gradient 6.96 -> 6.36 ms, its volume
// gradient 11.12 -> 10.94 ms.  On fp32 volumes of the 64-view 200^2
// workload the same split was slower than expm1f (forward 2.17 against 2.08
// ms), so they keep it.
template <typename T>
__device__ __forceinline__ float opacity(float x) {
    if constexpr (sizeof(T) == 2) {
        if (fabsf(x) < 0.125f) {
            const float p = fmaf(-0.2f * x, 1.0f, 1.0f);              // 1 - x/5
            const float q = fmaf(-0.25f * x, p, 1.0f);                // 1 - x/4 (...)
            const float r = fmaf(-(1.0f / 3.0f) * x, q, 1.0f);        // 1 - x/3 (...)
            const float t = fmaf(-0.5f * x, r, 1.0f);                 // 1 - x/2 (...)
            return x * t;
        }
        return 1.0f - __expf(-x);
    } else {
        return -expm1f(-x);
    }
}

template <typename T, bool GLOBAL = true>
__device__ __forceinline__ float trilinear_at(const T* __restrict__ base, int row, int slice,
                                              float fx, float fy, float fz) {
    auto ld = [](const T* p) { return GLOBAL ? load_voxel(p) : load_voxel_any(p); };
    const float v000 = ld(base);
    const float v100 = ld(base + 1);
    const float v010 = ld(base + row);
    const float v110 = ld(base + row + 1);
    const float v001 = ld(base + slice);
    const float v101 = ld(base + slice + 1);
    const float v011 = ld(base + slice + row);
    const float v111 = ld(base + slice + row + 1);
    const float c00 = fmaf(fx, v100 - v000, v000);
    const float c10 = fmaf(fx, v110 - v010, v010);
    const float c01 = fmaf(fx, v101 - v001, v001);
    const float c11 = fmaf(fx, v111 - v011, v011);
    const float c0 = fmaf(fy, c10 - c00, c00);
    const float c1 = fmaf(fy, c11 - c01, c01);
    return fmaf(fz, c1 - c0, c0);
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

// One sample in the xy-quad layout: the quads of slices k and k + 1 (voxels
// (i + a, j + b) at element a + 2b), the same scalar lerps as trilinear_at.
// fp32: two 16-byte loads; bf16: two 8-byte loads, widened exactly.
__device__ __forceinline__ void load_quad(const float* __restrict__ p, float v[4]) {
    const float4 q = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
}

__device__ __forceinline__ void load_quad(const uint16_t* __restrict__ p, float v[4]) {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = __uint_as_float(q.x << 16);
    v[1] = __uint_as_float(q.x & 0xFFFF0000u);
    v[2] = __uint_as_float(q.y << 16);
    v[3] = __uint_as_float(q.y & 0xFFFF0000u);
}

template <typename T>
__device__ __forceinline__ float sample_quads(const T* __restrict__ p, int slice, float fx,
                                              float fy, float fz) {
    float lo[4], hi[4];
    load_quad(p, lo);
    load_quad(p + 4 * (size_t)slice, hi);
    const float c00 = fmaf(fx, lo[1] - lo[0], lo[0]);
    const float c10 = fmaf(fx, lo[3] - lo[2], lo[2]);
    const float c01 = fmaf(fx, hi[1] - hi[0], hi[0]);
    const float c11 = fmaf(fx, hi[3] - hi[2], hi[2]);
    const float c0 = fmaf(fy, c10 - c00, c00);
    const float c1 = fmaf(fy, c11 - c01, c01);
    return fmaf(fz, c1 - c0, c0);
}

// One sample in the bricked layout: the 8 corners in one brick at constant
// offsets (kBrickEdge voxels per row, kBrickPlane per plane); the linear
// layout's loads and lerps.
template <typename T, bool GLOBAL = true>
__device__ __forceinline__ float sample_brick(const T* __restrict__ p, float fx, float fy,
                                              float fz) {
    return trilinear_at<T, GLOBAL>(p, kBrickEdge, kBrickPlane, fx, fy, fz);
}

}  // namespace
}  // namespace drr

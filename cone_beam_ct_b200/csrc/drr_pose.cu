// drr_pose.cu -- pose gradient of the DRR ray-march (sm_100a).
//
// dL/d[R|t] for L = sum over pixels of grad_out * image, the 12 entries of
// each view's world-to-camera matrix taken as free variables (flashdrr
// rendering API docs, VolumeRaycaster: rendering is differentiable with
// respect to the view matrices; the FlashDRR page's registration use).  The
// ray as written: direction R^T K^-1 (u, v, 1) normalised, centre -R^T t,
// clipped to the voxel-centre box, N midpoint samples, I = df * dt * sum mu.
//
// Differentiating the midpoint sum: with t_i = t0 + (i + 1/2) dt and
// p_i = C + t_i d (IJK),
//   dI = df [ d(dt) S + dt sum_i grad mu(p_i) . dp_i ],
//   dp_i = dC + t_i dd + (dt0 + (i + 1/2) d(dt)) d,
// so one pass along the ray needs only S = sum mu_i, G = sum grad mu_i and
// J = sum (i + 1/2) grad mu_i (fp32, like the forward's sum); everything
// after the loop -- the derivatives of the clip ends (each moves with the
// box plane it lies on; an entry point pinned at the camera does not move),
// of C = -R^T t and of the unit direction -- is per ray, in fp64, and
// folded into the 12 entries before a block reduction and one fp32 atomic
// add per entry and CTA.  grad mu is the gradient of the trilinear
// interpolant inside each sample's cell, from the same 8 corners the
// forward reads, so the loop is the forward's gather with about twice its
// arithmetic.  Batched calls (volumes x channels x views, the forward's
// batch rule) map each image to its pose and volume-channel; images that
// share a pose add into the same 12 entries.
#include <cuda_runtime.h>
#include <stdint.h>

#include "drr_internal.cuh"
#include "drr_sample.cuh"

namespace drr {
namespace {

__device__ __forceinline__ float widen(float v) { return v; }
__device__ __forceinline__ float widen(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

// The 8 corners of the sample's cell, corner (a, b, c) at v[a + 2b + 4c].
template <typename T, int LAYOUT>
__device__ __forceinline__ void cell_corners(const T* __restrict__ vol, const Geom& g, int cx,
                                             int cy, int cz, float v[8]) {
    if (!in_bounds(sample_offset<LAYOUT>(cell_index<LAYOUT>(g, cx, cy, cz)),
                   sample_extent<LAYOUT>(g), g.vstride)) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = 0.0f;
        return;
    }
    if (LAYOUT == 2) {
        const T* p = vol + (size_t)(cz * g.slice + cy * g.row + cx) * 8;
        if constexpr (sizeof(T) == 4) {
            const float4 lo = __ldg(reinterpret_cast<const float4*>(p));
            const float4 hi = __ldg(reinterpret_cast<const float4*>(p) + 1);
            v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
            v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
        } else {
            const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
            const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                v[2 * m] = __uint_as_float(words[m] << 16);
                v[2 * m + 1] = __uint_as_float(words[m] & 0xFFFF0000u);
            }
        }
    } else if (LAYOUT == 4) {
        const T* p = vol + brick_element(g, cx, cy, cz);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            v[e] = widen(__ldg(p + ((e & 1) ? 1 : 0) + ((e & 2) ? kBrickEdge : 0) +
                               ((e & 4) ? kBrickPlane : 0)));
    } else if (LAYOUT == 3) {
        const T* p = vol + (size_t)(cz * g.slice + cy * g.row + cx) * 4;
        load_quad(p, v);
        load_quad(p + 4 * (size_t)g.slice, v + 4);
    } else {
        const T* p = vol + (cz * g.slice + cy * g.row + cx);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            v[e] = widen(__ldg(p + ((e & 1) ? 1 : 0) + ((e & 2) ? g.row : 0) + ((e & 4) ? g.slice : 0)));
    }
}

// Value and gradient of the trilinear interpolant from a bf16 corner record,
// the forward's packed form (drr_sample.cuh): the a = 0 corners widened by a
// byte permute, the x differences by the mixed bf16 subtraction, and the
// lerps of the row pairs (c = 0, c = 1) at b = 0 and b = 1 as FFMA2 steps.
// Each lane computes what the scalar loop below computes, operation for
// operation.
__device__ __forceinline__ void value_grad_bf16(const uint16_t* __restrict__ p, float fx, float fy,
                                                float fz, float& val, float& gx, float& gy,
                                                float& gz) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
    const float2 lo0 = make_float2(__uint_as_float(__byte_perm(w.x, 0u, 0x1044)),
                                   __uint_as_float(__byte_perm(w.z, 0u, 0x1044)));
    const float2 lo1 = make_float2(__uint_as_float(__byte_perm(w.y, 0u, 0x1044)),
                                   __uint_as_float(__byte_perm(w.w, 0u, 0x1044)));
    const float2 d0 = make_float2(sub_bf16_f32((unsigned short)(w.x >> 16), lo0.x),
                                  sub_bf16_f32((unsigned short)(w.z >> 16), lo0.y));  // (d00, d01)
    const float2 d1 = make_float2(sub_bf16_f32((unsigned short)(w.y >> 16), lo1.x),
                                  sub_bf16_f32((unsigned short)(w.w >> 16), lo1.y));  // (d10, d11)
    const float2 m1 = make_float2(-1.0f, -1.0f);
    const float2 f2 = make_float2(fx, fx), fy2 = make_float2(fy, fy);
    const float2 x0 = __ffma2_rn(f2, d0, lo0);                 // (c00, c01)
    const float2 x1 = __ffma2_rn(f2, d1, lo1);                 // (c10, c11)
    const float2 e = __ffma2_rn(x0, m1, x1);                   // (e0, e1): y differences
    const float2 y = __ffma2_rn(fy2, e, x0);                   // (cy0, cy1)
    gz = y.y - y.x;
    val = fmaf(fz, gz, y.x);
    gy = fmaf(fz, e.y - e.x, e.x);
    const float2 dx = __ffma2_rn(fy2, __ffma2_rn(d0, m1, d1), d0);   // (dx0, dx1)
    gx = fmaf(fz, dx.y - dx.x, dx.x);
}

// Clip details of the ray through pixel (u, w), in fp64: the same arithmetic
// as ray_setup, keeping which axis each end of the clip lies on.
struct Clip {
    double C[3], d[3];          // IJK centre, IJK direction per mm
    double dw[3], q[3], nrm;    // unit world direction, K^-1 (u, w, 1), |R^T q|
    double t0, t1;
    int ax0, ax1;               // axes of the entry and exit planes
    bool pinned0;               // entry at the camera (t0 = 0): no derivative
};

__device__ __forceinline__ void clip_details(const View& v, const Geom& g, double u, double w,
                                             Clip& c) {
    c.q[0] = g.kinv[0] * u + g.kinv[1] * w + g.kinv[2];
    c.q[1] = g.kinv[3] * w + g.kinv[4];
    c.q[2] = g.kinv[5];
    double a[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) a[k] = v.A[3 * k] * u + v.A[3 * k + 1] * w + v.A[3 * k + 2];
    c.nrm = sqrt(a[0] * a[0] + a[1] * a[1] + a[2] * a[2]);
    const double rn = 1.0 / c.nrm;
    double t_near = -INFINITY, t_far = INFINITY;
    c.ax0 = -1;
    c.ax1 = -1;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        c.dw[k] = a[k] * rn;
        c.d[k] = a[k] * rn / g.spacing[k];
        c.C[k] = v.C[k];
        if (c.d[k] != 0.0) {
            const double ta = (0.0 - c.C[k]) / c.d[k];
            const double tb = ((double)g.hi[k] - c.C[k]) / c.d[k];
            const double tmin = fmin(ta, tb), tmax = fmax(ta, tb);
            if (tmin > t_near) {
                t_near = tmin;
                c.ax0 = k;
            }
            if (tmax < t_far) {
                t_far = tmax;
                c.ax1 = k;
            }
        }
    }
    c.pinned0 = !(t_near > 0.0);
    c.t0 = fmax(t_near, 0.0);
    c.t1 = t_far;
}

// acc[4r + c] += go * dI/dRt[r][c] for one ray, from its sums S, G, J.
__device__ __forceinline__ void pose_terms(const Clip& k, const Geom& g, const float* R12,
                                           float S, const float G[3], const float J[3], float go,
                                           double acc[12]) {
    const double N = (double)g.N, df = (double)g.density_factor;
    const double dt = (k.t1 - k.t0) / N;
    double Gd = 0.0, Jd = 0.0, gC[3], gd[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        Gd += (double)G[a] * k.d[a];
        Jd += (double)J[a] * k.d[a];
        gC[a] = df * dt * (double)G[a];
        gd[a] = df * dt * (k.t0 * (double)G[a] + dt * (double)J[a]);
    }
    const double kappa = df * ((double)S + dt * Jd) / N;   // per unit of d(t1) - d(t0)
    const double lambda = df * dt * Gd;                    // per unit of d(t0)
    // an end at t on the plane x_a = P moves by dt_end = -(dC_a + t dd_a) / d_a
    if (k.ax1 >= 0) {
        gC[k.ax1] -= kappa / k.d[k.ax1];
        gd[k.ax1] -= kappa * k.t1 / k.d[k.ax1];
    }
    if (!k.pinned0 && k.ax0 >= 0) {
        gC[k.ax0] -= (lambda - kappa) / k.d[k.ax0];
        gd[k.ax0] -= (lambda - kappa) * k.t0 / k.d[k.ax0];
    }
    // to world: C_ijk = (C_w - origin) / spacing, d_ijk = d_w / spacing
    double gCw[3], gdw[3], proj = 0.0;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        gCw[a] = gC[a] / g.spacing[a];
        gdw[a] = gd[a] / g.spacing[a];
        proj += gdw[a] * k.dw[a];
    }
    // d_w = R^T q / |R^T q|: dd_w/dR[r][c] = (I - d_w d_w^T) e_c q_r / |R^T q|
    // C_w = -R^T t:          dC_w/dR[r][c] = -t_r e_c,  dC_w/dt_r = -R[r][.]
    const double w = (double)go;
#pragma unroll
    for (int r = 0; r < 3; ++r) {
        const double tr = (double)R12[4 * r + 3], qn = k.q[r] / k.nrm;
        double gt = 0.0;
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            acc[4 * r + c] += w * (-tr * gCw[c] + qn * (gdw[c] - proj * k.dw[c]));
            gt -= (double)R12[4 * r + c] * gCw[c];
        }
        acc[4 * r + 3] += w * gt;
    }
}

// 4 CTAs per SM: caps the kernel at 64 registers.  The fp64 per-ray
// epilogue then spills (up to ~200 bytes, once per ray), the sample loop
// gains the occupancy; measured on B200 against 3 CTAs (80 registers): 3.95
// against 4.24 ms (256^3 bf16 corner records, 4 views of 1024^2 x 512),
// 2.29 against 2.49 ms (fp32 quads, 64 views of 200^2 x 256), 5.08 against
// 6.10 ms (512^3 fp32 corner records, 2 views of 2048^2 x 256).  (3 CTAs
// had beaten 2, 96 registers, 4.78 against 5.80 ms, before the packed bf16
// sample and the unroll.)
// BATCH: images map to poses and volume-channels by the batch rule (a
// separate instantiation, so that the single-volume kernel carries none of
// its registers).
template <typename T, int LAYOUT, int MODE, bool BATCH>
__global__ void __launch_bounds__(kThreads, 4)
pose_kernel(const T* __restrict__ vol_base, const float* __restrict__ Rt,
            const float* __restrict__ grad_out, const float* __restrict__ fwd_out,
            float* __restrict__ grad_Rt, const Geom g) {
    __shared__ View sv;
    __shared__ float sR[12];
    __shared__ double red[kThreads / 32][12];
    const int b = blockIdx.z;                    // output image (view x channel)
    const T* __restrict__ vol = BATCH ? vol_base + batch_item(g, b).slot * g.vstride : vol_base;
    if (!in_bounds(BATCH ? batch_item(g, b).slot * g.vstride : 0, g.vstride,
                   batch_slots(g) * g.vstride))
        return;
    {
        const int pose = BATCH ? batch_item(g, b).pose : b;
        if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)pose, g, sv);
        if (threadIdx.x < 12) sR[threadIdx.x] = Rt[12 * (size_t)pose + threadIdx.x];
    }
    __syncthreads();
    int r, c;
    tile_pixel(r, c);
    double acc[12];
#pragma unroll
    for (int e = 0; e < 12; ++e) acc[e] = 0.0;
    if (r < g.H && c < g.W) {
        const size_t pix = ((size_t)b * g.H + r) * g.W + c;
        float go = in_bounds(pix, 1, (long long)g.B * g.H * g.W) ? grad_out[pix] : 0.0f;
        if (MODE == 1) go *= 1.0f - fwd_out[pix];           // d(1 - e^-I)/dI = e^-I
        Ray ray;
        if (go != 0.0f && ray_setup(sv, g, (double)c, (double)r, LAYOUT == 1 ? 1.0 : 0.0, ray)) {
            // every sample in [0, g.lim], so every corner read is in the stored
            // volume (ray_setup); the gradient is the one inside that cell
            long long qx = ray.q0[0], qy = ray.q0[1], qz = ray.q0[2];
            float S = 0.0f, G2 = 0.0f, J2 = 0.0f, hi = 0.5f;          // hi = i + 1/2, exact
            float2 G01 = make_float2(0.0f, 0.0f), J01 = make_float2(0.0f, 0.0f);
            // alpha: s = df dt, the image C, and the running T_i and C_i
            const float sa = MODE == 2 ? g.density_factor * ray.dt : 0.0f;
            const float Cray = MODE == 2 ? fwd_out[pix] : 0.0f;
            float Tr = 1.0f, Ci = 0.0f;
            // unrolled by 2 (B200, 1024^2 x 512: 4.18 against 4.71 ms)
#pragma unroll 2
            for (int i = 0; i < g.N; ++i) {
                const float fx = fix_frac(qx), fy = fix_frac(qy), fz = fix_frac(qz);
                float val, gx, gy, gz;
                if constexpr (LAYOUT == 2 && sizeof(T) == 2) {
                    const int cell = fix_cell(qz) * g.slice + fix_cell(qy) * g.row + fix_cell(qx);
                    if (in_bounds((long long)cell * 8, 8, g.vstride)) {
                        value_grad_bf16(reinterpret_cast<const uint16_t*>(vol) + (size_t)cell * 8,
                                        fx, fy, fz, val, gx, gy, gz);
                    } else {
                        val = gx = gy = gz = 0.0f;
                    }
                } else {
                    float v[8];
                    cell_corners<T, LAYOUT>(vol, g, fix_cell(qx), fix_cell(qy), fix_cell(qz), v);
                    const float d00 = v[1] - v[0], d10 = v[3] - v[2];   // x differences, rows (b, c)
                    const float d01 = v[5] - v[4], d11 = v[7] - v[6];
                    const float c00 = fmaf(fx, d00, v[0]), c10 = fmaf(fx, d10, v[2]);
                    const float c01 = fmaf(fx, d01, v[4]), c11 = fmaf(fx, d11, v[6]);
                    const float e0 = c10 - c00, e1 = c11 - c01;         // y differences
                    const float cy0 = fmaf(fy, e0, c00), cy1 = fmaf(fy, e1, c01);
                    gz = cy1 - cy0;
                    gy = fmaf(fz, e1 - e0, e0);
                    const float dx0 = fmaf(fy, d10 - d00, d00), dx1 = fmaf(fy, d11 - d01, d01);
                    gx = fmaf(fz, dx1 - dx0, dx0);
                    val = fmaf(fz, gz, cy0);
                }
                qx += ray.s[0];
                qy += ray.s[1];
                qz += ray.s[2];
                if constexpr (MODE == 2) {
                    // dC/dmu_i = T_i (s (1 - a_i) mu_i + a_i) - s (C - C_i) weights the
                    // sample's gradient; S collects dC/ds = sum T_i mu_i^2 (1 - a_i)
                    // - mu_i (C - C_i) (a_i = 1 - exp(-s mu_i), as the forward)
                    const float a = opacity<T>(sa * val);
                    const float keep = 1.0f - a;
                    Ci = fmaf(Tr * a, val, Ci);
                    const float rest = Cray - Ci;
                    const float wgt = Tr * fmaf(sa * keep, val, a) - sa * rest;
                    S += fmaf(Tr * val * keep, val, -val * rest);
                    Tr *= keep;
                    gx *= wgt;
                    gy *= wgt;
                    gz *= wgt;
                } else {
                    S += val;
                }
                G01 = __fadd2_rn(G01, make_float2(gx, gy));
                G2 += gz;
                J01 = __ffma2_rn(make_float2(hi, hi), make_float2(gx, gy), J01);
                J2 = fmaf(hi, gz, J2);
                hi += 1.0f;
            }
            float G[3] = {G01.x, G01.y, G2}, J[3] = {J01.x, J01.y, J2};
            if constexpr (MODE == 2) {
                // sum_i w_i grad mu_i . dp_i is the line integral's df dt sum with
                // G, J divided by df dt (pose_terms multiplies them back); S
                // enters as dC/ds with ds = df d(dt), as S does for the integral
                const float inv = sa != 0.0f ? 1.0f / sa : 0.0f;
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    G[a] *= inv;
                    J[a] *= inv;
                }
            }
            Clip k;
            clip_details(sv, g, (double)c, (double)r, k);
            pose_terms(k, g, sR, S, G, J, go, acc);
        }
    }
    // block sum of the 12 entries (fp64), then one fp32 atomic add per entry
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int e = 0; e < 12; ++e) {
        double x = acc[e];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_down_sync(0xffffffffu, x, off);
        if (lane == 0) red[warp][e] = x;
    }
    __syncthreads();
    if (threadIdx.x < 12) {
        double x = 0.0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) x += red[w][threadIdx.x];
        const int pose = BATCH ? batch_item(g, blockIdx.z).pose : (int)blockIdx.z;
        const long long poses = g.broadcast ? 1 : g.B / g.C;
        if (x != 0.0 && in_bounds(12LL * pose + threadIdx.x, 1, 12 * poses))
            atomicAdd(grad_Rt + 12 * (size_t)pose + threadIdx.x, (float)x);
    }
}

template <typename T, int LAYOUT>
cudaError_t launch_typed(const void* vol, const Geom& g, const float* Rt, int mode,
                         const float* grad_out, const float* fwd_out, float* grad_Rt,
                         cudaStream_t stream) {
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    const T* v = static_cast<const T*>(vol);
    const bool batch = g.C != 1 || g.broadcast || g.views_per_vol != g.B;
#define DRR_POSE_LAUNCH(M, BT) \
    pose_kernel<T, LAYOUT, M, BT><<<grid, kThreads, 0, stream>>>(v, Rt, grad_out, fwd_out, grad_Rt, g)
    if (batch) {
        if (mode == 2) DRR_POSE_LAUNCH(2, true);
        else if (mode == 1) DRR_POSE_LAUNCH(1, true);
        else DRR_POSE_LAUNCH(0, true);
    } else {
        if (mode == 2) DRR_POSE_LAUNCH(2, false);
        else if (mode == 1) DRR_POSE_LAUNCH(1, false);
        else DRR_POSE_LAUNCH(0, false);
    }
#undef DRR_POSE_LAUNCH
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_layout(const void* vol, int layout, const Geom& g, const float* Rt, int mode,
                          const float* grad_out, const float* fwd_out, float* grad_Rt,
                          cudaStream_t stream) {
    if (layout == 4) return launch_typed<T, 4>(vol, g, Rt, mode, grad_out, fwd_out, grad_Rt, stream);
    if (layout == 3) return launch_typed<T, 3>(vol, g, Rt, mode, grad_out, fwd_out, grad_Rt, stream);
    if (layout == 2) return launch_typed<T, 2>(vol, g, Rt, mode, grad_out, fwd_out, grad_Rt, stream);
    if (layout == 1) return launch_typed<T, 1>(vol, g, Rt, mode, grad_out, fwd_out, grad_Rt, stream);
    return launch_typed<T, 0>(vol, g, Rt, mode, grad_out, fwd_out, grad_Rt, stream);
}

}  // namespace

DRR_BOUNDS_READER(bounds_word_pose)

cudaError_t launch_pose_grad(const void* vol, int dtype, int layout, const Geom& g,
                             const float* Rt, int mode, const float* grad_out,
                             const float* fwd_out, float* grad_Rt, cudaStream_t stream) {
    if (dtype == 0)
        return launch_layout<float>(vol, layout, g, Rt, mode, grad_out, fwd_out, grad_Rt, stream);
    return launch_layout<uint16_t>(vol, layout, g, Rt, mode, grad_out, fwd_out, grad_Rt, stream);
}

}  // namespace drr

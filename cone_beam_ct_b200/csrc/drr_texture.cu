// drr_texture.cu -- the texture-trilinear comparison (include/drr_texture.h).
//
// Not the product path: the same ray-march as drr_forward.cu with the
// trilinear interpolation done by the texture units (tex3D, linear filter,
// zero border, unnormalised coordinates at texel centres), which weights the
// 8 corners with 8-bit fixed-point fractions (TorchTomo page, "Fast CUDA
// Kernels").  One texture fetch per sample replaces 8 gathers and 7 lerps;
// the comparison measures what that costs in accuracy.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <new>

#include "../../include/drr_texture.h"
#include "drr_internal.cuh"

struct drr_tex_volume {
    cudaArray_t array;
    cudaTextureObject_t tex;
    int dims[3];
    int texel;
};

namespace {

thread_local char g_err[512] = "";

int fail(int rc, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return rc;
}

int cuda_rc(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return 0;
    return fail((int)e, "%s: %s", what, cudaGetErrorString(e));
}

__global__ void to_half(const float* __restrict__ src, __half* __restrict__ dst, int64_t n) {
    for (int64_t m = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; m < n;
         m += (int64_t)gridDim.x * blockDim.x)
        dst[m] = __float2half_rn(src[m]);
}

template <int MODE>
__global__ void __launch_bounds__(drr::kThreads)
tex_forward_kernel(cudaTextureObject_t tex, const float* __restrict__ Rt, float* __restrict__ out,
                   const drr::Geom g) {
    __shared__ drr::View sv;
    const int b = blockIdx.z;
    if (threadIdx.x == 0) drr::view_setup(Rt + 12 * (size_t)b, g, sv);
    __syncthreads();
    int r, c;
    drr::tile_pixel(r, c);
    if (r >= g.H || c >= g.W) return;
    drr::Ray ray;
    float result = 0.0f;
    if (drr::ray_setup(sv, g, (double)c, (double)r, 0.0, ray)) {
        // texel centres sit at integer + 0.5 in unnormalised texture coordinates
        const double inv = 1.0 / drr::kFix;
        const float x0 = (float)(ray.q0[0] * inv + 0.5), sx = (float)(ray.s[0] * inv);
        const float y0 = (float)(ray.q0[1] * inv + 0.5), sy = (float)(ray.s[1] * inv);
        const float z0 = (float)(ray.q0[2] * inv + 0.5), sz = (float)(ray.s[2] * inv);
        float acc = 0.0f, fi = 0.0f;
#pragma unroll 4
        for (int i = 0; i < g.N; ++i, fi += 1.0f)
            acc += tex3D<float>(tex, fmaf(fi, sx, x0), fmaf(fi, sy, y0), fmaf(fi, sz, z0));
        const float I = (g.density_factor * ray.dt) * acc;
        result = (MODE == 1) ? -expm1f(-I) : I;
    }
    out[((size_t)b * g.H + r) * g.W + c] = result;
}

}  // namespace

extern "C" {

DRR_TEX_API const char* drr_tex_last_error(void) { return g_err; }

DRR_TEX_API int drr_tex_create(const float* vol, const int dims[3], int texel,
                               drr_tex_volume** out) {
    if (!vol || !dims || !out) return fail(-1, "vol, dims and out must be non-NULL");
    if (texel != 0 && texel != 1) return fail(-1, "texel must be 0 (float32) or 1 (float16)");
    for (int a = 0; a < 3; ++a)
        if (dims[a] < 2 || dims[a] > 16384) return fail(-1, "dims[%d] out of [2, 16384]", a);
    *out = nullptr;
    drr_tex_volume* t = new (std::nothrow) drr_tex_volume();
    if (!t) return fail(-1, "out of host memory");
    t->dims[0] = dims[0];
    t->dims[1] = dims[1];
    t->dims[2] = dims[2];
    t->texel = texel;
    const size_t n = (size_t)dims[0] * dims[1] * dims[2];
    cudaChannelFormatDesc desc = texel == 0 ? cudaCreateChannelDesc<float>()
                                            : cudaCreateChannelDescHalf();
    const cudaExtent ext = make_cudaExtent(dims[0], dims[1], dims[2]);
    int rc = cuda_rc(cudaMalloc3DArray(&t->array, &desc, ext), "cudaMalloc3DArray");
    void* staged = nullptr;
    if (!rc && texel == 1) {
        rc = cuda_rc(cudaMalloc(&staged, n * sizeof(__half)), "cudaMalloc");
        if (!rc) {
            to_half<<<148 * 8, 256>>>(vol, static_cast<__half*>(staged), (int64_t)n);
            rc = cuda_rc(cudaGetLastError(), "to_half launch");
        }
    }
    if (!rc) {
        cudaMemcpy3DParms p = {};
        const size_t elem = texel == 0 ? sizeof(float) : sizeof(__half);
        p.srcPtr = make_cudaPitchedPtr(texel == 0 ? const_cast<float*>(vol) : staged,
                                       dims[0] * elem, dims[0], dims[1]);
        p.dstArray = t->array;
        p.extent = ext;
        p.kind = cudaMemcpyDeviceToDevice;
        rc = cuda_rc(cudaMemcpy3D(&p), "cudaMemcpy3D");
    }
    if (staged) cudaFree(staged);
    if (!rc) {
        cudaResourceDesc res = {};
        res.resType = cudaResourceTypeArray;
        res.res.array.array = t->array;
        cudaTextureDesc td = {};
        for (int a = 0; a < 3; ++a) td.addressMode[a] = cudaAddressModeBorder;   // zero outside
        td.filterMode = cudaFilterModeLinear;
        td.readMode = cudaReadModeElementType;
        td.normalizedCoords = 0;
        rc = cuda_rc(cudaCreateTextureObject(&t->tex, &res, &td, nullptr), "cudaCreateTextureObject");
    }
    if (!rc) rc = cuda_rc(cudaDeviceSynchronize(), "texture upload");
    if (rc) {
        if (t->array) cudaFreeArray(t->array);
        delete t;
        return rc;
    }
    *out = t;
    return 0;
}

DRR_TEX_API int drr_tex_render(const drr_tex_volume* t, const float spacing[3],
                               const float origin[3], const float K[9], const float* Rt, int B,
                               int H, int W, int n_samples, float density_factor, int mode,
                               float* out, void* stream) {
    if (!t || !spacing || !origin || !K || !Rt || !out) return fail(-1, "NULL argument");
    if (B < 1 || B > 65535 || H < 1 || H > 65535 * drr::kTileH || W < 1 || n_samples < 1 ||
        n_samples > (1 << 20) || (mode != 0 && mode != 1) || !std::isfinite(density_factor))
        return fail(-1, "invalid sizes, mode or density_factor");
    for (int a = 0; a < 3; ++a)
        if (!(spacing[a] > 0.0f) || !std::isfinite(spacing[a]) || !std::isfinite(origin[a]))
            return fail(-1, "invalid spacing or origin");
    if (K[3] != 0.0f || K[6] != 0.0f || K[7] != 0.0f || K[0] == 0.0f || K[4] == 0.0f ||
        K[8] == 0.0f)
        return fail(-1, "K must be upper triangular and invertible");
    drr::Geom g;
    drr::fill_geom(g, t->dims, spacing, origin, K, B, H, W, n_samples, density_factor, 0);
    const dim3 grid((W + drr::kTileW - 1) / drr::kTileW, (H + drr::kTileH - 1) / drr::kTileH, B);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (mode == 1)
        tex_forward_kernel<1><<<grid, drr::kThreads, 0, s>>>(t->tex, Rt, out, g);
    else
        tex_forward_kernel<0><<<grid, drr::kThreads, 0, s>>>(t->tex, Rt, out, g);
    return cuda_rc(cudaGetLastError(), "tex_forward_kernel launch");
}

DRR_TEX_API int drr_tex_destroy(drr_tex_volume* t) {
    if (!t) return 0;
    int rc = cuda_rc(cudaDeviceSynchronize(), "drr_tex_destroy sync");
    cudaDestroyTextureObject(t->tex);
    cudaFreeArray(t->array);
    delete t;
    return rc;
}

}  // extern "C"

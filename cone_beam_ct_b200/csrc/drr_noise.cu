// drr_noise.cu -- the Gaussian-Poisson surrogate of shot noise and its
// derivative (flashdrr.rendering API docs, VolumeRaycaster.apply_poisson:
// Gaussian noise of standard deviation sqrt(transmission / i0) added to the
// transmission, clamped to [0, 1]; a differentiable stand-in for Poisson
// noise).  Applied here to a Beer-Lambert image 1 - T: the transmission is
// T = 1 - image and the result is 1 - T', T' = clamp(T + sqrt(T / i0) z, 0, 1),
// with the standard normal draws z supplied by the caller.  Elementwise and
// bound by HBM: grid-stride loops over coalesced fp32 arrays.
#include <cuda_runtime.h>
#include <stdint.h>

#include "drr_internal.cuh"

namespace drr {
namespace {

__global__ void __launch_bounds__(256)
poisson_noise_kernel(const float* __restrict__ image, const float* __restrict__ z, float i0,
                     float* out, int64_t n) {
    for (int64_t m = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; m < n;
         m += (int64_t)gridDim.x * blockDim.x) {
        const float T = 1.0f - image[m];
        float Tn = T > 0.0f ? fmaf(sqrtf(T / i0), z[m], T) : T;
        Tn = fminf(fmaxf(Tn, 0.0f), 1.0f);
        out[m] = 1.0f - Tn;
    }
}

// d out / d image = dT'/dT = 1 + z / (2 sqrt(T i0)) where the clamp is
// inactive (0 < T + sqrt(T / i0) z < 1) and T > 0, else 0.
__global__ void __launch_bounds__(256)
poisson_noise_backward_kernel(const float* __restrict__ image, const float* __restrict__ z,
                              float i0, const float* __restrict__ grad_out,
                              float* __restrict__ grad_image, int64_t n) {
    for (int64_t m = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; m < n;
         m += (int64_t)gridDim.x * blockDim.x) {
        const float T = 1.0f - image[m];
        float slope = 0.0f;
        if (T > 0.0f) {
            const float zm = z[m];
            const float Tn = fmaf(sqrtf(T / i0), zm, T);
            if (Tn > 0.0f && Tn < 1.0f) slope = 1.0f + zm / (2.0f * sqrtf(T * i0));
        }
        grad_image[m] = grad_out[m] * slope;
    }
}

int grid_for_elements(int64_t n) {
    const int64_t blocks = (n + 255) / 256;
    const int64_t cap = 148 * 8;
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

// (the elementwise loops index only [0, n): nothing to check)
DRR_BOUNDS_READER(bounds_word_noise)

cudaError_t launch_poisson_noise(const float* image, const float* z, float i0, float* out,
                                 int64_t n, cudaStream_t stream) {
    poisson_noise_kernel<<<grid_for_elements(n), 256, 0, stream>>>(image, z, i0, out, n);
    return cudaGetLastError();
}

cudaError_t launch_poisson_noise_backward(const float* image, const float* z, float i0,
                                          const float* grad_out, float* grad_image, int64_t n,
                                          cudaStream_t stream) {
    poisson_noise_backward_kernel<<<grid_for_elements(n), 256, 0, stream>>>(image, z, i0, grad_out,
                                                                           grad_image, n);
    return cudaGetLastError();
}

}  // namespace drr

// drr_probe.cu -- L2 read-bandwidth probe for the gather roofline
// (include/drr_probe.h).  Grid-stride float4 loads with the .cg cache
// operator (cached in L2, not in L1), one persistent wave of CTAs (4 of 512
// threads per SM).
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/drr_probe.h"

namespace {

__global__ void __launch_bounds__(512) l2_read(const float4* __restrict__ buf, size_t n, int reps,
                                               float* __restrict__ sink) {
    float acc = 0.0f;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (int r = 0; r < reps; ++r) {
        size_t m = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
        // 4 independent loads in flight per thread (measured on B200 over
        // 64 MiB: 19.4 TB/s, against 18.3 with one)
        for (; m + 3 * stride < n; m += 4 * stride) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = __ldcg(buf + m + u * stride);
#pragma unroll
            for (int u = 0; u < 4; ++u) acc += (v[u].x + v[u].y) + (v[u].z + v[u].w);
        }
        for (; m < n; m += stride) {
            const float4 v = __ldcg(buf + m);
            acc += (v.x + v.y) + (v.z + v.w);
        }
    }
    if (acc != acc) *sink = acc;   // never true for finite data
}

}  // namespace

extern "C" DRR_PROBE_API int drr_probe_l2_read(const void* buf, size_t n_vec16, int reps,
                                               float* sink, void* stream) {
    if (!buf || !sink || n_vec16 == 0 || reps < 1 ||
        (reinterpret_cast<uintptr_t>(buf) % 16) != 0)
        return -1;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    l2_read<<<sms * 4, 512, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const float4*>(buf), n_vec16, reps, sink);
    return (int)cudaGetLastError();
}

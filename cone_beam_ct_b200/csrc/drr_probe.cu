// drr_probe.cu -- the benchmark's probes (include/drr_probe.h): the L2 read
// bandwidth of the gather roofline (grid-stride float4 loads with the .cg
// cache operator, cached in L2, not in L1; one persistent wave of CTAs, 4 of
// 512 threads per SM), and the L2's fp32 reduction (RED) throughput beside
// which the adjoint's scatter is read.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/drr_probe.h"
#include "drr_barrier.cuh"

namespace {

// Self-test of the grid barrier: every CTA passes `rounds` barriers that
// expect `expected` arrivals each and counts the ones it got through.  With
// expected above the grid's CTA count no epoch completes: the first wait
// that runs out raises the abort word and the others leave.
__global__ void __launch_bounds__(256) barrier_probe(unsigned* bar, unsigned expected,
                                                     unsigned long long timeout_ns, int rounds,
                                                     unsigned long long* timeouts, int* passes) {
    unsigned epoch = 0;
    int n = 0;
    for (int r = 0; r < rounds; ++r) {
        if (!drr::grid_barrier(bar, epoch, expected, timeout_ns, timeouts)) break;
        ++n;
    }
    if (threadIdx.x == 0) atomicAdd(passes, n);
}

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

// fp32 reductions over an L2-resident buffer, one persistent wave; every pass
// adds 1 to each float the pattern touches:
//   kind 0  scalar, a warp's 32 lanes on 32 consecutive floats (each 32-byte
//           sector receives one operation carrying 8 values)
//   kind 1  16-byte vector, each lane on its own 32-byte record, two vector
//           reductions per record (each sector receives two operations of 4
//           values: the adjoint's corner-record flush)
//   kind 2  scalar, each lane on the first float of its own sector (one
//           operation carrying 1 value per sector: scattered adds)
__global__ void __launch_bounds__(512) l2_red(float* __restrict__ buf, size_t n, int reps,
                                              int kind) {
    const size_t tid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (int r = 0; r < reps; ++r) {
        if (kind == 0) {
            for (size_t m = tid; m < n; m += stride) atomicAdd(buf + m, 1.0f);
        } else if (kind == 1) {
            for (size_t m = tid; m < n / 8; m += stride) {
                float4* p = reinterpret_cast<float4*>(buf + 8 * m);
                atomicAdd(p, make_float4(1.0f, 1.0f, 1.0f, 1.0f));
                atomicAdd(p + 1, make_float4(1.0f, 1.0f, 1.0f, 1.0f));
            }
        } else {
            for (size_t m = tid; m < n / 8; m += stride) atomicAdd(buf + 8 * m, 1.0f);
        }
    }
}

}  // namespace

extern "C" DRR_PROBE_API int drr_probe_l2_red(float* buf, size_t n_floats, int reps, int kind,
                                              void* stream) {
    if (!buf || n_floats < 8 || (n_floats % 8) != 0 || reps < 1 || kind < 0 || kind > 2 ||
        (reinterpret_cast<uintptr_t>(buf) % 32) != 0)
        return -1;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    l2_red<<<sms * 4, 512, 0, static_cast<cudaStream_t>(stream)>>>(buf, n_floats, reps, kind);
    return (int)cudaGetLastError();
}

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

extern "C" DRR_PROBE_API int drr_probe_grid_barrier(int extra_arrivals, int rounds,
                                                    double timeout_ms,
                                                    unsigned long long* timeouts_out,
                                                    int* passes_out, int* ctas_out) {
    if (extra_arrivals < 0 || rounds < 1 || rounds > 4096 || !(timeout_ms > 0.0) ||
        timeout_ms > 60000.0 || !timeouts_out || !passes_out || !ctas_out)
        return -1;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return (int)e;
    struct Words {
        unsigned bar[4];
        unsigned long long timeouts;
        int passes;
    };
    Words* w = nullptr;
    e = cudaMalloc(&w, sizeof(Words));
    if (e != cudaSuccess) return (int)e;
    e = cudaMemset(w, 0, sizeof(Words));
    unsigned* bar = w->bar;
    unsigned expected = (unsigned)(sms + extra_arrivals);
    unsigned long long timeout_ns = (unsigned long long)(timeout_ms * 1e6);
    unsigned long long* timeouts = &w->timeouts;
    int* passes = &w->passes;
    void* args[] = {(void*)&bar, (void*)&expected, (void*)&timeout_ns, (void*)&rounds,
                    (void*)&timeouts, (void*)&passes};
    // one CTA per SM, launched cooperatively: all resident
    if (e == cudaSuccess)
        e = cudaLaunchCooperativeKernel((const void*)barrier_probe, dim3(sms), dim3(256), args, 0,
                                        0);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    Words h{};
    if (e == cudaSuccess) e = cudaMemcpy(&h, w, sizeof(Words), cudaMemcpyDeviceToHost);
    cudaFree(w);
    if (e != cudaSuccess) return (int)e;
    *timeouts_out = h.timeouts;
    *passes_out = h.passes;
    *ctas_out = sms;
    return 0;
}

// drr_barrier.cuh -- a bounded grid-wide barrier for cooperative launches
// (sm_100a): the sparse views' slab pass of the volume adjoint separates its
// phases with it, and the probe library's self-test drives it (including a
// wait that runs out).
#pragma once

#include <cuda_runtime.h>

namespace drr {

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Grid-wide barrier over a cooperative launch (every CTA resident), reused
// epoch after epoch within one launch.  bar[0] counts arrivals over the
// launch (epoch e is complete at e * expected arrivals: `expected` is the
// grid's CTA count), bar[1] holds the last released epoch, bar[2] is the
// abort word; all three start at 0.  A wait that lasts timeout_ns raises the
// abort word, so that every other CTA leaves at its next wait, and adds 1
// to *timeouts.  Returns false if this or another CTA gave up (the caller
// returns: the work after the barrier is abandoned).
__device__ inline bool grid_barrier(unsigned* bar, unsigned& epoch, unsigned expected,
                                    unsigned long long timeout_ns,
                                    unsigned long long* timeouts) {
    __shared__ int s_ok;
    __syncthreads();
    ++epoch;
    if (threadIdx.x == 0) {
        volatile unsigned* vb = bar;
        int ok = vb[2] == 0u;
        if (ok) {
            __threadfence();                     // this CTA's writes before its arrival
            const unsigned arrived = atomicAdd(&bar[0], 1u) + 1u;
            if (arrived == epoch * expected) {
                __threadfence();
                atomicExch(&bar[1], epoch);
            } else {
                const unsigned long long t0 = global_ns();
                while (vb[1] < epoch) {
                    if (vb[2] != 0u) {
                        ok = 0;
                        break;
                    }
                    if (global_ns() - t0 > timeout_ns) {
                        atomicExch(&bar[2], 1u);
                        atomicAdd(timeouts, 1ull);
                        ok = 0;
                        break;
                    }
                    __nanosleep(256);
                }
            }
            __threadfence();                     // the other CTAs' writes before ours
        }
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

}  // namespace drr

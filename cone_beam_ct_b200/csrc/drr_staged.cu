// drr_staged.cu -- forward ray-march of the bricked layout with each layer of
// a tile's frustum staged in shared memory by the TMA engine (sm_100a).
//
// The volume-layout subsystem's "optional TMA staging of volume bricks into
// shared memory for narrow frusta": the rays of a 16 x 16 pixel tile form a
// narrow pyramid, and where the rays are about a voxel apart or sparser
// (many views of a small detector) the samples of neighbouring rays share
// few cache lines, so gathers from L2 and DRAM dominate with long latency.
// Here the CTA walks its pyramid one layer of bricks at a time along the
// major axis m of its central ray.  Before the rays sample layer L, one
// thread copies the bricks of layer L that the pyramid crosses (at most
// kStageBricks; the lateral window comes from the tile's 4 corner rays,
// which bound every ray of the tile) from global into shared memory with
// bulk copies (cp.async.bulk, completion counted in bytes on an mbarrier);
// the copies of layer L + 1 go into the other of two buffers while the rays
// sample layer L.  A sample reads its 8 corners from the staged brick -- the
// bricked layout keeps a cell's corners in one brick -- with the same lerps
// as the global path, so staged and global samples give the same bits.  A
// sample whose brick is not staged (a layer wider than the window, a ray
// leaving it) reads global memory.
//
// Waits are bounded: if a layer's copies do not complete within kWaitTries
// tries of the mbarrier, the thread reads that layer from global memory, the
// CTA stages nothing more, and before it exits one thread waits (bounded
// again) for the copies still in flight.  The results are those of the
// global path either way.
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>

#include "drr_internal.cuh"
#include "drr_sample.cuh"

namespace drr {
namespace {

constexpr int kStageBricks = 16;                 // bricks of one staged layer (4 x 4 laterally)
constexpr unsigned kWaitTries = 1u << 16;        // mbarrier tries before a wait gives up
constexpr int kPlanLayers = 128;                 // layers planned (later ones read global memory)
constexpr double kStageMinVoxels = 8.0;          // tile width at the volume centre worth staging

// PTX wrappers: shared-memory addresses are 32-bit offsets in the CTA's window.
__device__ __forceinline__ unsigned smem_u32(const void* p) {
    return (unsigned)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned arrivals) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(arrivals)
                 : "memory");
}

// make the initialised barriers visible to the asynchronous (copy) proxy
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// one arrival that also announces `bytes` of copies to complete this phase
__device__ __forceinline__ void mbar_arrive_expect(unsigned long long* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// one try at the phase with this parity (the hardware may hold the thread a
// while inside a try); true once that phase has completed
__device__ __forceinline__ bool mbar_try(unsigned long long* bar, unsigned parity) {
    unsigned done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long* bar, unsigned parity) {
    for (unsigned n = 0; n < kWaitTries; ++n)
        if (mbar_try(bar, parity)) return true;
    return false;
}

// bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// global memory into this CTA's shared memory (the CTA's own window: the
// kernel is not launched as a cluster), counted on `bar`
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes,
                                         unsigned long long* bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"((unsigned long long)__cvta_generic_to_global(src)), "r"(bytes),
        "r"(smem_u32(bar))
        : "memory");
}

// order this thread's earlier generic-proxy shared-memory accesses (the
// CTA's reads, made visible to it by a barrier) before later copies into
// the same bytes
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// A staged layer: bricks [a0, a0 + na) x [b0, b0 + nb) (the two lateral
// axes) of brick layer L along m, in buffer slots ib * na + ia; `staged`
// says whether the copies were issued, `parity` which phase of the buffer's
// barrier completes them.
struct Layer {
    int L, a0, b0, na, nb, staged, parity;
};

// the tile's 4 corner rays (C and d in IJK) and the axes of its pyramid
struct Frustum {
    double C[3];
    double d[4][3];
    int m, dir;                  // major axis of the central ray, its direction (+1 / -1)
    int nbricks[3];              // bricks per axis
};

template <int M>
struct Axes {                    // the lateral axes of major axis M, ascending
    static constexpr int A = M == 0 ? 1 : 0;
    static constexpr int B = M == 2 ? 1 : 2;
};

// Lateral brick window of brick layer L (cells [8L, 8L + 8) along m) over the
// 4 corner rays at the layer's two bounding planes.
__device__ __forceinline__ void layer_window(const Frustum& f, int L, int& a0, int& b0, int& na,
                                             int& nb) {
    const int m = f.m, A = m == 0 ? 1 : 0, B = m == 2 ? 1 : 2;
    double lo_a = INFINITY, hi_a = -INFINITY, lo_b = INFINITY, hi_b = -INFINITY;
    bool ok = true;
    for (int j = 0; j < 4; ++j) {
        const double dm = f.d[j][m];
        ok = ok && fabs(dm) > 1e-12;
        for (int side = 0; side < 2; ++side) {
            const double t = ((double)(kBrick * (L + side)) - f.C[m]) / dm;
            const double pa = f.C[A] + t * f.d[j][A], pb = f.C[B] + t * f.d[j][B];
            lo_a = fmin(lo_a, pa);
            hi_a = fmax(hi_a, pa);
            lo_b = fmin(lo_b, pb);
            hi_b = fmax(hi_b, pb);
        }
    }
    // a margin far above the fixed-point positions' rounding (2^-32 voxel)
    const double eps = 1e-3;
    if (!ok || !(fabs(lo_a) < 1e8 && fabs(hi_a) < 1e8 && fabs(lo_b) < 1e8 && fabs(hi_b) < 1e8)) {
        na = nb = 0;
        a0 = b0 = 0;
        return;
    }
    const int ca0 = (int)floor(lo_a - eps), ca1 = (int)floor(hi_a + eps);
    const int cb0 = (int)floor(lo_b - eps), cb1 = (int)floor(hi_b + eps);
    a0 = max(ca0 >> 3, 0);
    b0 = max(cb0 >> 3, 0);
    const int a1 = min(ca1 >> 3, f.nbricks[A] - 1), b1 = min(cb1 >> 3, f.nbricks[B] - 1);
    na = max(a1 - a0 + 1, 0);
    nb = max(b1 - b0 + 1, 0);
}

// Record layer L (window w = a0, b0, na, nb) in `lay` and, if the window
// fits, issue its copies into buffer `buf` (one thread).
template <typename T>
__device__ __forceinline__ void stage_layer(const Frustum& f, const Geom& g, const T* vol, T* stage,
                                            unsigned long long* bar, Layer& lay, int L, int4 w,
                                            int buf, int& uses, bool stop) {
    const int a0 = w.x, b0 = w.y, na = w.z, nb = w.w;
    const int m = f.m;
    lay.L = L;
    lay.a0 = a0;
    lay.b0 = b0;
    lay.na = na;
    lay.nb = nb;
    lay.staged = 0;
    lay.parity = uses & 1;
    const long long total = (long long)f.nbricks[0] * f.nbricks[1] * f.nbricks[2];
    if (stop || na < 1 || nb < 1 || na * nb > kStageBricks || L < 0 || L >= f.nbricks[m]) return;
    constexpr unsigned kBytes = kBrickStride * sizeof(T);
    static_assert(kBytes % 16 == 0, "bulk copies move multiples of 16 bytes");
    // every copy's source brick, checked before any is issued: inside the
    // stored bricks, both ends 16-byte aligned (else the layer is not staged)
    long long src[kStageBricks];
    for (int n = 0; n < na * nb; ++n) {
        const int ia = n % na, ib = n / na;
        const int cm = L, ca = a0 + ia, cb = b0 + ib;
        const int cx = m == 0 ? cm : ca, cy = m == 1 ? cm : (m == 0 ? ca : cb), cz = m == 2 ? cm : cb;
        const long long brick = ((long long)cz * f.nbricks[1] + cy) * f.nbricks[0] + cx;
        const T* sp = vol + brick * kBrickStride;
        const T* dp = stage + ((size_t)buf * kStageBricks + n) * kBrickStride;
        if (brick < 0 || brick >= total ||
            !in_bounds(brick * kBrickStride, kBrickStride, g.vstride) ||
            (reinterpret_cast<uintptr_t>(sp) & 15) != 0 || (smem_u32(dp) & 15) != 0)
            return;
        src[n] = brick;
    }
    mbar_arrive_expect(bar + buf, kBytes * (unsigned)(na * nb));
    for (int n = 0; n < na * nb; ++n)
        bulk_g2s(stage + ((size_t)buf * kStageBricks + n) * kBrickStride,
                 vol + src[n] * kBrickStride, kBytes, bar + buf);
    lay.staged = 1;
    ++uses;
}

// The samples of one ray in brick layer lay.L (and any earlier in the walk's
// direction: a ray sampled out of order reads global memory): from the
// staged bricks where the window holds them.  Returns when the next sample
// lies beyond the layer, or at the end of the ray.
template <typename T, int M>
__device__ __forceinline__ void sample_layer(const T* __restrict__ vol, const T* __restrict__ buf,
                                             const Geom& g, const Layer& lay, bool use, int dir,
                                             long long q[3], const long long s[3], int& i,
                                             float& acc) {
    constexpr int A = Axes<M>::A, B = Axes<M>::B;
    while (i < g.N) {
        const int c[3] = {fix_cell(q[0]), fix_cell(q[1]), fix_cell(q[2])};
        const int lm = c[M] >> 3;
        if (dir > 0 ? lm > lay.L : lm < lay.L) return;
        const float fx = fix_frac_fs(q[0]), fy = fix_frac_fs(q[1]), fz = fix_frac_fs(q[2]);
        const int ia = (c[A] >> 3) - lay.a0, ib = (c[B] >> 3) - lay.b0;
        if (use && lm == lay.L && (unsigned)ia < (unsigned)lay.na && (unsigned)ib < (unsigned)lay.nb) {
            const int local = ((c[2] & 7) * kBrickEdge + (c[1] & 7)) * kBrickEdge + (c[0] & 7);
            // a shared-memory brick: ordinary loads (not the global read-only path)
            acc += sample_brick<T, false>(buf + (ib * lay.na + ia) * kBrickStride + local, fx, fy,
                                          fz);
        } else {
            const int e = brick_element(g, c[0], c[1], c[2]);
            if (in_bounds(e, sample_extent<4>(g), g.vstride)) acc += sample_brick(vol + e, fx, fy, fz);
        }
        q[0] += s[0];
        q[1] += s[1];
        q[2] += s[2];
        ++i;
    }
}

template <typename T, int MODE>
__global__ void __launch_bounds__(kThreads)
forward_staged_kernel(const T* __restrict__ vol_base, const float* __restrict__ Rt,
                      float* __restrict__ out, const Geom g) {
    extern __shared__ __align__(128) unsigned char stage_raw[];
    T* const stage = reinterpret_cast<T*>(stage_raw);   // [2][kStageBricks][kBrickStride]
    __shared__ View sv;
    __shared__ Frustum fr;
    __shared__ __align__(8) unsigned long long bar[2];
    __shared__ Layer lay[2];
    __shared__ int4 s_win[kPlanLayers];          // each layer's window, planned in parallel
    __shared__ int s_lmin, s_lmax, s_fail, s_uses[2], s_stage;
    const int b = blockIdx.z;
    const BatchItem it = batch_item(g, b);
    if (!in_bounds(it.slot * g.vstride, g.vstride, batch_slots(g) * g.vstride)) return;
    const T* __restrict__ vol = vol_base + it.slot * g.vstride;
    const int tid = threadIdx.x;
    if (tid == 0) {
        view_setup(Rt + 12 * (size_t)it.pose, g, sv);
        // the central ray's IJK direction picks the walk's axis; the 4 corner
        // pixels' rays bound the tile's pyramid
        const double u0 = blockIdx.x * kTileW, v0 = blockIdx.y * kTileH;
        double dc[3], big = -1.0;
        int m = 0;
        for (int k = 0; k < 3; ++k) {
            const double a = sv.A[3 * k] * (u0 + 0.5 * (kTileW - 1)) +
                             sv.A[3 * k + 1] * (v0 + 0.5 * (kTileH - 1)) + sv.A[3 * k + 2];
            dc[k] = a / g.spacing[k];
            if (fabs(dc[k]) > big) {
                big = fabs(dc[k]);
                m = k;
            }
            fr.C[k] = sv.C[k];
        }
        fr.m = m;
        fr.dir = dc[m] >= 0.0 ? 1 : -1;
        for (int j = 0; j < 4; ++j) {
            const double u = u0 + ((j & 1) ? kTileW - 1 : 0), v = v0 + ((j & 2) ? kTileH - 1 : 0);
            for (int k = 0; k < 3; ++k)
                fr.d[j][k] = (sv.A[3 * k] * u + sv.A[3 * k + 1] * v + sv.A[3 * k + 2]) / g.spacing[k];
        }
        // stage only sparse tiles: where the tile spans at least kStageMinVoxels
        // voxels at the volume centre (rays about a voxel apart or more), dense
        // rays reuse each voxel through L1 and a barrier per layer costs more
        // than staging saves (B200, 1024^2 and 2048^2 C-arm views: 2-3.5x
        // slower staged)
        double cc2 = 0.0, n0 = 0.0, n1 = 0.0, dot = 0.0;
        for (int k = 0; k < 3; ++k) {
            const double off = (fr.C[k] - 0.5 * g.hi[k]) * g.spacing[k];
            const double w0 = fr.d[0][k] * g.spacing[k], w1 = fr.d[1][k] * g.spacing[k];
            cc2 += off * off;
            n0 += w0 * w0;
            n1 += w1 * w1;
            dot += w0 * w1;
        }
        const double ang = acos(fmin(1.0, fmax(-1.0, dot / sqrt(n0 * n1))));
        const double min_sp = fmin(g.spacing[0], fmin(g.spacing[1], g.spacing[2]));
        s_stage = (sqrt(cc2) * ang / min_sp) >= kStageMinVoxels ? 1 : 0;
        fr.nbricks[0] = brick_count(g.nx);
        fr.nbricks[1] = brick_count(g.ny);
        fr.nbricks[2] = brick_count(g.nz);
        s_lmin = INT_MAX;
        s_lmax = INT_MIN;
        s_fail = 0;
        s_uses[0] = s_uses[1] = 0;
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_init_fence();
    }
    __syncthreads();

    int r, c;
    tile_pixel(r, c);
    const bool in_image = r < g.H && c < g.W;
    Ray ray;
    const bool hit = in_image && ray_setup(sv, g, (double)c, (double)r, 0.0, ray);
    long long q[3] = {0, 0, 0}, s[3] = {0, 0, 0};
    int i = hit ? 0 : g.N;
    float acc = 0.0f;
    const int m = fr.m, dir = fr.dir;
    if (hit) {
        for (int k = 0; k < 3; ++k) {
            q[k] = ray.q0[k];
            s[k] = ray.s[k];
        }
    }
    if (s_stage) {
        int lo = INT_MAX, hi = INT_MIN;
        if (hit) {
            // (selects, not q[m]: a runtime index would put q and s in local memory)
            const long long qm = m == 0 ? q[0] : m == 1 ? q[1] : q[2];
            const long long sm = m == 0 ? s[0] : m == 1 ? s[1] : s[2];
            const int l0 = fix_cell(qm) >> 3, l1 = fix_cell(qm + (long long)(g.N - 1) * sm) >> 3;
            lo = min(l0, l1);
            hi = max(l0, l1);
        }
        lo = __reduce_min_sync(0xFFFFFFFFu, lo);
        hi = __reduce_max_sync(0xFFFFFFFFu, hi);
        if ((tid & 31) == 0 && lo <= hi) {
            atomicMin(&s_lmin, lo);
            atomicMax(&s_lmax, hi);
        }
        __syncthreads();
        const int lmin = s_lmin, lmax = s_lmax;
        // 0: no ray of the tile hits the volume
        const int nl = lmin <= lmax ? min(lmax - lmin + 1, kPlanLayers) : 0;
        auto layer_of = [&](int k) { return dir > 0 ? lmin + k : lmax - k; };
        // every layer's window at once, one thread per layer
        if (tid < nl) {
            int4 w;
            layer_window(fr, layer_of(tid), w.x, w.y, w.z, w.w);
            s_win[tid] = w;
        }
        __syncthreads();
        if (tid == 0 && nl > 0)
            stage_layer(fr, g, vol, stage, bar, lay[0], layer_of(0), s_win[0], 0, s_uses[0], false);
        __syncthreads();
        for (int k = 0; k < nl; ++k) {
            const int buf = k & 1;
            if (tid == 0 && k + 1 < nl) {
                // buffer buf ^ 1 was last read in layer k - 1, which every thread
                // finished before the barrier that ended it
                fence_proxy_async();
                stage_layer(fr, g, vol, stage, bar, lay[buf ^ 1], layer_of(k + 1), s_win[k + 1],
                            buf ^ 1, s_uses[buf ^ 1], s_fail != 0);
            }
            const Layer L = lay[buf];
            bool use = L.staged != 0;
            if (use && !mbar_wait_bounded(&bar[buf], (unsigned)L.parity)) {
                use = false;                          // read this layer from global memory
                atomicOr(&s_fail, 1);                 // and stage nothing more
            }
            const T* sbuf = stage + (size_t)buf * kStageBricks * kBrickStride;
            if (m == 0)
                sample_layer<T, 0>(vol, sbuf, g, L, use, dir, q, s, i, acc);
            else if (m == 1)
                sample_layer<T, 1>(vol, sbuf, g, L, use, dir, q, s, i, acc);
            else
                sample_layer<T, 2>(vol, sbuf, g, L, use, dir, q, s, i, acc);
            __syncthreads();
        }
    }
    // a dense tile's rays, and samples left over by the walk (none for rays
    // monotone along m, none past kPlanLayers layers): global memory
    if (i < g.N) {
        Layer none{dir > 0 ? INT_MAX : INT_MIN, 0, 0, 0, 0, 0, 0};
        sample_layer<T, 0>(vol, stage, g, none, false, dir, q, s, i, acc);
    }
    // after a wait gave up, copies may still be landing in this CTA's shared
    // memory: wait for the last phase of each buffer (bounded) before exiting
    if (tid == 0 && s_fail) {
        for (int bb = 0; bb < 2; ++bb)
            if (s_uses[bb] > 0) mbar_wait_bounded(&bar[bb], (unsigned)((s_uses[bb] - 1) & 1));
    }
    if (!in_image) return;
    float result = 0.0f;
    if (hit) {
        const float I = (g.density_factor * ray.dt) * acc;
        result = MODE == 1 ? -expm1f(-I) : I;
    }
    const long long pix = ((long long)b * g.H + r) * g.W + c;
    if (in_bounds(pix, 1, (long long)g.B * g.H * g.W)) out[pix] = result;
}

template <typename T>
cudaError_t launch_staged_typed(const void* vol, const Geom& g, const float* Rt, int mode,
                                float* out, cudaStream_t stream) {
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    const size_t smem = 2 * kStageBricks * kBrickStride * sizeof(T);
    const T* v = static_cast<const T*>(vol);
    cudaError_t e;
    if (mode == 1) {
        e = cudaFuncSetAttribute(forward_staged_kernel<T, 1>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        forward_staged_kernel<T, 1><<<grid, kThreads, smem, stream>>>(v, Rt, out, g);
    } else {
        e = cudaFuncSetAttribute(forward_staged_kernel<T, 0>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        forward_staged_kernel<T, 0><<<grid, kThreads, smem, stream>>>(v, Rt, out, g);
    }
    return cudaGetLastError();
}

}  // namespace

DRR_BOUNDS_READER(bounds_word_staged)

cudaError_t launch_forward_staged(const void* vol, int dtype, const Geom& g, const float* Rt,
                                  int mode, float* out, cudaStream_t stream) {
    if (dtype == 0) return launch_staged_typed<float>(vol, g, Rt, mode, out, stream);
    return launch_staged_typed<uint16_t>(vol, g, Rt, mode, out, stream);
}

}  // namespace drr

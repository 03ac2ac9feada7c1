// drr_adjoint.cu -- adjoint (volume gradient) of the DRR ray-march (sm_100a).
//
// The transpose of the forward operator (TorchTomo page, "Discrete Adjoint
// and Learned Primal-Dual": <A x, y> = <x, A^T y>): every sample of every
// ray scatters g * w_corner into the 8 voxels its trilinear interpolation
// read, with g = grad_out * density_factor * dt per ray, times exp(-I) =
// 1 - out in Beer-Lambert mode (the derivative of 1 - exp(-I)).  This is the
// backward kernel of the fused renderer (FlashDRR page, "Train vs. Eval
// Dynamics").  Same ray setup and 32.32 sample positions as the forward on
// the linear layout, so its weights are the forward's weights and the
// adjoint is that forward's transpose up to fp32 rounding.
//
// Where the time goes: the fp32 atomic adds, which the L2 executes at a fixed
// rate of sector operations, and which stall on hot spots when many rays
// cross the same voxels at once.  Three measures cut both:
//  * A pending block per ray: the 8 corner sums of the current cell stay in
//    registers while consecutive samples fall into overlapping cells; when
//    the cell moves by one along an axis only the face that leaves is
//    flushed (4 atomics) and the rest slides over.  Per sample the ray then
//    issues ~4 (|S_x| + |S_y| + |S_z|) atomics instead of 8 (S: the step in
//    voxels), the fewer the denser the sampling.
//  * Phases: each warp of the grid starts its rays at a different eighth of
//    their length (wrapping round), so that warps working on neighbouring
//    rays at the same time are at different depths rather than on the same
//    voxels.
//  * Lane mapping by density: where a 16 x 16 pixel tile spans fewer than 8
//    voxels (rays much closer than a voxel), lanes are spread over the whole
//    tile so that the lanes of one atomic instruction hit different words;
//    otherwise a warp keeps an 8 x 4 block of neighbouring rays, whose
//    atomics share sectors.
// Measured alternatives (shared-memory windows flushed with coalesced global
// atomics; no pending block; no phases) were slower on every workload.
//
// With a workspace (drr_render_adjoint_ws), views whose rays are much closer
// than a voxel ("dense": where a 16-pixel tile spans fewer than 8 voxels at
// the volume centre) accumulate instead into corner records: for every cell
// its 8 corner sums, contiguous (32 bytes, one L2 sector).  A 3 x 2 bundle
// of neighbouring rays keeps the records of its current cells pending in
// registers and flushes one, when the bundle leaves that cell, with two
// 16-byte vector atomics -- the L2 executes a vector atomic at the same rate
// as a scalar one, so this carries 4x the payload per operation, and the
// bundle flushes once where its rays would have flushed up to six times.  A
// record sums the moments of its samples (records_kernel); a scatter pass
// then turns each record into corner weights and adds them to the gradient
// volume.  The alpha gradient (its per-sample factor in place of the ray's
// scale) and batched calls (records per volume-channel) take the same path.
//
// The sparse views of a call with a workspace accumulate into records too,
// but one slab of cell layers at a time, each slab's records small enough to
// stay in the L2 (slab_adjoint_kernel): the whole record array gained
// nothing there (12-20 ms against the direct path's 9.3 on the 256^3 volume
// seen by 64 views of 200^2, the records going to DRAM between views), the
// slabs take 6.7 ms.  Without a workspace every view takes the direct path.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "drr_barrier.cuh"
#include "drr_internal.cuh"
#include "drr_sample.cuh"

namespace drr {

// Built-in scratch of drr_render_adjoint_noalloc, for callers that may not
// allocate device memory.  It is part of the library's device image: every
// GPU that loads the library holds these bytes until the process exits.
// Host code must not use this name as an address (on the host it is only a
// stand-in); noalloc_scratch() below fetches the device address.
static __device__ __align__(256) unsigned char noalloc_scratch_bytes[kNoAllocScratchBytes];

namespace {

// 8 corner sums of a pending block at cell (x, y, z); a[k] belongs to corner
// (k & 1, (k >> 1) & 1, k >> 2).
// (n: elements of the gradient volume at grad, for the bounds-checked build)
__device__ __forceinline__ void flush_block(float* __restrict__ grad, const int st[3],
                                            const int cell[3], const float a[8], long long n) {
    const int base = cell[2] * st[2] + cell[1] * st[1] + cell[0];
    float* p = grad + base;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int off = ((k & 1) ? 1 : 0) + ((k & 2) ? st[1] : 0) + ((k & 4) ? st[2] : 0);
        if (in_bounds(base + off, 1, n)) atomicAdd(p + off, a[k]);
    }
}

// Move the pending block one cell along axis AX (d = +1 or -1): flush the face
// that leaves, slide the other face over, start the new face at zero.
template <int AX>
__device__ __forceinline__ void slide(int d, float* __restrict__ grad, const int st[3], int cell[3],
                                      float a[8], long long nvox) {
    if (d == 0) return;
    const int side = d > 0 ? 0 : 1;                           // face that leaves
    constexpr int A = AX == 0 ? 1 : 0, B = AX == 2 ? 1 : 2;   // the other two axes, ascending
    const int base = (cell[2] * st[2] + cell[1] * st[1] + cell[0]) + (side ? st[AX] : 0);
    float* p = grad + base;
    float v[4];
    int n = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (((k >> AX) & 1) == 0) v[n++] = side ? a[k | (1 << AX)] : a[k];
    if (in_bounds(base, 1, nvox)) atomicAdd(p, v[0]);
    if (in_bounds(base + st[A], 1, nvox)) atomicAdd(p + st[A], v[1]);
    if (in_bounds(base + st[B], 1, nvox)) atomicAdd(p + st[B], v[2]);
    if (in_bounds(base + st[A] + st[B], 1, nvox)) atomicAdd(p + st[A] + st[B], v[3]);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (((k >> AX) & 1) != 0) continue;
        const int hi = k | (1 << AX);
        if (d > 0) {
            a[k] = a[hi];
            a[hi] = 0.0f;
        } else {
            a[hi] = a[k];
            a[k] = 0.0f;
        }
    }
    cell[AX] += d;
}

// Is a 16-pixel tile at pixel (u0, v0) narrower than 8 voxels where its rays
// cross the volume centre?  (NaN geometry: no.)
__device__ __forceinline__ bool dense_tile(const View& v, const Geom& g, double u0, double v0) {
    double c2 = 0.0, n0 = 0.0, n1 = 0.0, dot = 0.0;
    for (int k = 0; k < 3; ++k) {
        const double d0 = v.A[3 * k] * u0 + v.A[3 * k + 1] * v0 + v.A[3 * k + 2];
        const double d1 = d0 + v.A[3 * k] * (double)kTileW;
        const double off = (v.C[k] - 0.5 * g.hi[k]) * g.spacing[k];   // camera to centre, mm
        c2 += off * off;
        n0 += d0 * d0;
        n1 += d1 * d1;
        dot += d0 * d1;
    }
    const double ang = acos(fmin(1.0, fmax(-1.0, dot / sqrt(n0 * n1))));
    const double min_sp = fmin(g.spacing[0], fmin(g.spacing[1], g.spacing[2]));
    return (sqrt(c2) * ang / min_sp) < 8.0;
}

// Fire-and-forget fp32 reductions into global memory, spelled out so that
// they are L2 reductions whatever the compiler can prove about the pointer
// (an add it cannot place in global memory becomes a generic atomic that
// waits for its old value: the slab pass took 9.6 instead of 6.8 ms).  No memory
// clobber: nothing in a kernel reads what these add before a barrier or a
// fence, which order them for the compiler.
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(__cvta_generic_to_global(p)),
                 "f"(a), "f"(b), "f"(c), "f"(d));
}
__device__ __forceinline__ void red_add(float* p, float a) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(__cvta_generic_to_global(p)), "f"(a));
}

// Flush a pending corner record: two 16-byte vector reductions into one
// sector.  (n: floats of the record array at rec, for the bounds-checked
// build)
__device__ __forceinline__ void flush_record(float* __restrict__ rec, int cell, const float2 a[4],
                                             long long n) {
    if (!in_bounds((long long)cell * 8, 8, n)) return;
    float* p = rec + (size_t)cell * 8;
    red_add_v4(p, a[0].x, a[0].y, a[1].x, a[1].y);
    red_add_v4(p + 4, a[2].x, a[2].y, a[3].x, a[3].y);
}

// Workspace layout (drr_render_adjoint_ws, header_layout below): a header
// of ints -- [0] bit 0 "some view is dense", bit 1 "some view is sparse";
// [1 + b] "view b is dense" (b: output image) -- then, 16-byte aligned, the
// slab pass's grid-barrier words, then, 256-byte aligned, every view's View
// (K^-1 R^T and camera centre, written by plan_views); then, 256-byte
// aligned, the corner records of each volume-channel slot, 8 floats per
// cell, cell = (k * (ny-1) + j) * (nx-1) + i.  The sparse views' slabs
// (slab_adjoint_kernel) reuse the start of the record area once the dense
// views' records are scattered.
constexpr int kSomeDense = 1, kSomeSparse = 2;
struct HeaderLayout {
    size_t bar, views, rec;                      // byte offsets
};
__host__ __device__ inline HeaderLayout header_layout(int B) {
    const size_t bar = ((size_t)(1 + B) * sizeof(int) + 15) / 16 * 16;
    const size_t views = (bar + 4 * sizeof(unsigned) + 255) / 256 * 256;
    const size_t rec = (views + (size_t)B * sizeof(View) + 255) / 256 * 256;
    return {bar, views, rec};
}

struct Workspace {
    int* flags;        // NULL: no workspace, every view takes the direct path
    float* rec;        // records of volume-channel slot 0; slot s at rec + s * rec_stride
    long long rec_stride;
    // the record kernel's 16 warp phases are spread over 2^-phase_shift of
    // the ray's length (see launch_adjoint)
    int phase_shift;
    unsigned* bar;     // grid barrier: [0] arrivals, [1] released epoch, [2] abort
    const View* views;
};

// Which views accumulate into records: one CTA loops over the views, so
// that flags[0] is written once, after all of them.  It also stores each
// view's View and clears the barrier words for the slab pass.
__global__ void __launch_bounds__(256) plan_views(const float* __restrict__ Rt, const Geom g,
                                                  int* __restrict__ flags,
                                                  View* __restrict__ views,
                                                  unsigned* __restrict__ bar) {
    __shared__ int any;
    if (threadIdx.x == 0) {
        any = 0;
        for (int k = 0; k < 4; ++k) bar[k] = 0u;
    }
    __syncthreads();
    int mine = 0;
    for (int b = threadIdx.x; b < g.B; b += blockDim.x) {
        View v;
        view_setup(Rt + 12 * (size_t)batch_item(g, b).pose, g, v);
        views[b] = v;
        // a view is judged by its first tile: every tile subtends nearly the
        // same angle (the pixel pitch is constant across the detector)
        const int dense = dense_tile(v, g, 0.0, 0.0) ? 1 : 0;
        flags[1 + b] = dense;
        mine |= dense ? kSomeDense : kSomeSparse;
    }
    if (mine) atomicOr(&any, mine);
    __syncthreads();
    if (threadIdx.x == 0) flags[0] = any;
}

// Zero n4 float4 of records when some view will use them (flags[0] & use).
__global__ void zero_records(const int* __restrict__ flags, int use, float4* __restrict__ rec,
                             int64_t n4) {
    if ((flags[0] & use) == 0) return;
    const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int64_t m = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; m < n4;
         m += (int64_t)gridDim.x * blockDim.x)
        rec[m] = z;
}

// Records written as moments (records_kernel) into the gradient volume: each
// cell's 8 moments become its 8 corner weights (per axis, the pair
// (sum s g, sum s g f) becomes (sum s g (1 - f), sum s g f); x, then y, then
// z), which are added to the cell's 8 corner voxels with atomic adds.  A CTA
// takes whole x rows of cells (one division per row for (j, k) and the
// volume-channel slot); consecutive threads hold consecutive cells, so each
// of the 8 adds of a warp covers 32 consecutive voxels (4 or 5 L2 sectors).
// Zero weights are skipped.
__device__ __forceinline__ void moments_to_corner_weights(float v[8]) {
#pragma unroll
    for (int axis = 0; axis < 3; ++axis) {
        const int st = 1 << axis;
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if ((e & st) == 0) v[e] -= v[e | st];
    }
}

__global__ void scatter_records(const int* __restrict__ flags, const float* __restrict__ rec,
                                long long rec_stride, float* __restrict__ grad, int nx, int ny,
                                int nz, int slots) {
    if ((flags[0] & kSomeDense) == 0) return;
    const int crow = nx - 1, rows = (ny - 1) * (nz - 1);    // cells per row, rows per slot
    const long long total = (long long)rows * slots;
    const long long nxy = (long long)nx * ny, nvox = nxy * nz;
    for (long long row = blockIdx.x; row < total; row += gridDim.x) {
        const int slot = (int)(row / rows);
        const int rr = (int)(row - (long long)slot * rows);
        const int k = rr / (ny - 1), j = rr - k * (ny - 1);
        const float4* __restrict__ r =
            reinterpret_cast<const float4*>(rec + slot * rec_stride + (long long)rr * crow * 8);
        float* __restrict__ gr = grad + slot * nvox + k * nxy + (long long)j * nx;
        for (int i = threadIdx.x; i < crow; i += blockDim.x) {
            if (!in_bounds(((long long)rr * crow + i) * 8, 8, rec_stride)) continue;
            const float4 lo = __ldcs(r + 2 * i), hi = __ldcs(r + 2 * i + 1);
            float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            moments_to_corner_weights(v);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const long long off = i + (e & 1) + ((e >> 1) & 1) * nx + (e >> 2) * nxy;
                if (v[e] != 0.0f && in_bounds(k * nxy + (long long)j * nx + off, 1, nvox))
                    atomicAdd(gr + off, v[e]);
            }
        }
    }
}

// The direct path: every view without a workspace, or the views the plan
// left sparse (a CTA of a dense view returns at once -- a uniform exit before
// any barrier -- since records_kernel handles it).
template <int MODE>
__global__ void __launch_bounds__(kThreads)
adjoint_kernel(const float* __restrict__ Rt, const float* __restrict__ grad_out,
               const float* __restrict__ fwd_out, float* __restrict__ grad, const Geom g,
               const Workspace ws) {
    __shared__ View sv;
    __shared__ int s_dense;
    const int b = blockIdx.z;                    // output image (view x channel)
    const int tid = threadIdx.x;
    if (ws.flags != nullptr && ws.flags[1 + b] != 0) return;
    const BatchItem it = batch_item(g, b);
    if (!in_bounds(it.slot * g.vstride, g.vstride, batch_slots(g) * g.vstride)) return;
    grad += it.slot * g.vstride;                 // this volume-channel's gradient
    if (tid == 0) {
        view_setup(Rt + 12 * (size_t)it.pose, g, sv);
        s_dense = dense_tile(sv, g, blockIdx.x * kTileW, blockIdx.y * kTileH) ? 1 : 0;
    }
    __syncthreads();

    int r, c;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (s_dense) {
        // spread: the 32 lanes of a warp cover the whole 16 x 16 tile (bijective)
        c = blockIdx.x * kTileW + (lane & 7) * 2 + (warp & 1);
        r = blockIdx.y * kTileH + (lane >> 3) * 4 + (warp >> 1);
    } else {
        tile_pixel(r, c);
    }
    if (r >= g.H || c >= g.W) return;
    const size_t pix = ((size_t)b * g.H + r) * g.W + c;
    if (!in_bounds(pix, 1, (long long)g.B * g.H * g.W)) return;
    float go = grad_out[pix];
    if (MODE == 1) go *= 1.0f - fwd_out[pix];
    Ray ray;
    if (go == 0.0f || !ray_setup(sv, g, (double)c, (double)r, 0.0, ray)) return;
    const float scale = go * (g.density_factor * ray.dt);
    const int st[3] = {1, g.row, g.slice};

    // phase: this warp starts at sample `start` and wraps round to 0
    const int ph = (warp + blockIdx.x * 3 + blockIdx.y * 5 + blockIdx.z) & 7;
    const int start = (int)(((long long)g.N * ph) >> 3);

    int cell[3];
    float a[8];
    for (int pass = 0; pass < 2; ++pass) {
        const int i0 = pass == 0 ? start : 0;
        const int i1 = pass == 0 ? g.N : start;
        if (i0 >= i1) continue;
        long long qx = ray.q0[0] + (long long)i0 * ray.s[0];
        long long qy = ray.q0[1] + (long long)i0 * ray.s[1];
        long long qz = ray.q0[2] + (long long)i0 * ray.s[2];
        cell[0] = fix_cell(qx);
        cell[1] = fix_cell(qy);
        cell[2] = fix_cell(qz);
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = 0.0f;
        for (int i = i0; i < i1; ++i) {
            const int cx = fix_cell(qx), cy = fix_cell(qy), cz = fix_cell(qz);
            const int dx = cx - cell[0], dy = cy - cell[1], dz = cz - cell[2];
            if (dx < -1 || dx > 1 || dy < -1 || dy > 1 || dz < -1 || dz > 1) {
                // a step of more than one cell: flush the whole block and restart
                flush_block(grad, st, cell, a, g.vstride);
#pragma unroll
                for (int k = 0; k < 8; ++k) a[k] = 0.0f;
                cell[0] = cx;
                cell[1] = cy;
                cell[2] = cz;
            } else {
                slide<0>(dx, grad, st, cell, a, g.vstride);
                slide<1>(dy, grad, st, cell, a, g.vstride);
                slide<2>(dz, grad, st, cell, a, g.vstride);
            }
            const float fx = fix_frac(qx), fy = fix_frac(qy), fz = fix_frac(qz);
            const float wz1 = scale * fz, wz0 = scale * (1.0f - fz);
            const float w00 = wz0 * (1.0f - fy), w01 = wz0 * fy;
            const float w10 = wz1 * (1.0f - fy), w11 = wz1 * fy;
            const float gx = 1.0f - fx;
            a[0] += w00 * gx;
            a[1] += w00 * fx;
            a[2] += w01 * gx;
            a[3] += w01 * fx;
            a[4] += w10 * gx;
            a[5] += w10 * fx;
            a[6] += w11 * gx;
            a[7] += w11 * fx;
            qx += ray.s[0];
            qy += ray.s[1];
            qz += ray.s[2];
        }
        flush_block(grad, st, cell, a, g.vstride);
    }
}

// Record path for the views the plan marked dense.  A CTA covers a 48 x 32
// pixel tile; each thread owns a 3 x 2 bundle of neighbouring rays (less than
// a voxel across where this path runs) and two pending record slots, home to
// the bundle's upper and lower row.  A ray adds its sample to any slot
// already holding its cell, else flushes its home slot and takes it over, so
// a bundle that moves together flushes once per cell instead of once per
// ray.  A warp's bundles are neighbours (a 4 x 8 block of them) and warps
// start at one of 16 phases of the ray.  Measured on the 1024^2 x 512 and
// 2048^2 x 256 C-arm workloads (B200): neighbouring bundles beat bundles
// spread over the tile (7.1 vs 7.8 ms); 3 x 2 bundles flush 11 % less than
// 2 x 2 (0.26 against 0.30 flushes per ray-sample) and run 3 % / 8 % faster;
// a least-recently-used slot choice flushes less still but its extra
// branches doubled the issued instructions.  Letting a miss share the home
// slot's add (two divergent paths instead of three) took 7.12 to 6.65 ms at
// 1024^2 x 512, and packed fp32x2 weights and sums then 6.55 ms; summing
// the 8 trilinear moments instead of the 8 weights (fewer multiplies per
// sample, converted at flush) was slower (6.83 ms), and a third, victim slot much
// slower (8.6 ms, spills; 11.0 ms at 149 registers and 1 CTA per SM).
//
// A record accumulates the moments of its samples, not their weights: for a
// sample with fractions (fx, fy, fz) in its cell and ray scale s, entry
// a + 2b + 4c adds s fx^a fy^b fz^c.  The 8 trilinear weights are a fixed
// linear map of these (w_0 = 1 - f, w_1 = f per axis), applied once per
// record by scatter_records after the scatter, so a sample costs one
// multiply and three packed fp32x2 multiplies instead of the weights'
// products.
constexpr int kBundleX = 3, kBundleY = 2;        // rays per bundle, across and down
constexpr int kBundleRays = kBundleX * kBundleY;
constexpr int kSlots = 2;
constexpr int kRecTileW = 16 * kBundleX, kRecTileH = 16 * kBundleY;   // 48 x 32 pixels per CTA

template <int MODE>
__global__ void __launch_bounds__(kThreads, 2)
records_kernel(const float* __restrict__ Rt, const float* __restrict__ grad_out,
               const float* __restrict__ fwd_out, const Geom g, const Workspace ws) {
    __shared__ View sv;
    const int b = blockIdx.z;
    if (ws.flags[1 + b] == 0) return;            // sparse view: adjoint_kernel's
    const BatchItem it = batch_item(g, b);
    if (!in_bounds(it.slot * ws.rec_stride, ws.rec_stride, batch_slots(g) * ws.rec_stride)) return;
    float* const rec = ws.rec + it.slot * ws.rec_stride;   // this volume-channel's records
    if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)it.pose, g, sv);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a warp's 32 bundles form a 4 x 8 block of the 16 x 16 bundle grid (12 x
    // 16 rays; 8 x 4 bundles, 24 x 8 rays, measured 1 % slower)
    const int px = (warp & 3) * 4 + (lane & 3), py = (warp >> 2) * 8 + (lane >> 2);
    const int c0 = blockIdx.x * kRecTileW + px * kBundleX, r0 = blockIdx.y * kRecTileH + py * kBundleY;
    const int ph = (warp + blockIdx.x * 3 + blockIdx.y * 5 + blockIdx.z) & 15;   // 16 phases
    const int start = (int)(((long long)g.N * ph) >> ws.phase_shift);

    // per ray: its position at the current sample (32.32) and step; the start
    // of the second pass is recovered from the position after the first
    bool act[kBundleRays];
    float scale[kBundleRays];
    long long q[kBundleRays][3], s[kBundleRays][3];
#pragma unroll
    for (int k = 0; k < kBundleRays; ++k) {
        const int c = c0 + (k % kBundleX), r = r0 + (k / kBundleX);
        act[k] = false;
        scale[k] = 0.0f;
#pragma unroll
        for (int a = 0; a < 3; ++a) q[k][a] = s[k][a] = 0;
        if (r >= g.H || c >= g.W) continue;
        const size_t pix = ((size_t)b * g.H + r) * g.W + c;
        if (!in_bounds(pix, 1, (long long)g.B * g.H * g.W)) continue;
        float go = grad_out[pix];
        if (MODE == 1) go *= 1.0f - fwd_out[pix];
        Ray ray;
        if (go == 0.0f || !ray_setup(sv, g, (double)c, (double)r, 0.0, ray)) continue;
        act[k] = true;
        scale[k] = go * (g.density_factor * ray.dt);
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            s[k][a] = ray.s[a];
            q[k][a] = ray.q0[a] + (long long)start * ray.s[a];
        }
    }
    // cells stay in [0, n-2] per axis (linear-layout lim), inside the records
    const int cr = g.nx - 1, cs = (g.nx - 1) * (g.ny - 1);
    float2 p[kSlots][4];
    int pc[kSlots];
    for (int pass = 0; pass < 2; ++pass) {
        const int i0 = pass == 0 ? start : 0;
        const int i1 = pass == 0 ? g.N : start;
        if (pass == 1) {                         // back to sample 0: q0 = q(N) - N * s
#pragma unroll
            for (int k = 0; k < kBundleRays; ++k)
#pragma unroll
                for (int a = 0; a < 3; ++a) q[k][a] -= (long long)g.N * s[k][a];
        }
        if (i0 >= i1) continue;
#pragma unroll
        for (int h = 0; h < kSlots; ++h) pc[h] = -1;
        for (int i = i0; i < i1; ++i) {
#pragma unroll
            for (int k = 0; k < kBundleRays; ++k) {
                if (!act[k]) continue;
                const int cell = fix_cell(q[k][2]) * cs + fix_cell(q[k][1]) * cr + fix_cell(q[k][0]);
                const float fx = fix_frac(q[k][0]), fy = fix_frac(q[k][1]), fz = fix_frac(q[k][2]);
#pragma unroll
                for (int a = 0; a < 3; ++a) q[k][a] += s[k][a];
                // the sample's 8 moments s fx^a fy^b fz^c, as pairs (a = 0, 1):
                // one FMUL and three packed FMUL2
                const float2 mx = make_float2(scale[k], scale[k] * fx);
                const float2 mxy = __fmul2_rn(mx, make_float2(fy, fy));
                const float2 w[4] = {mx, mxy, __fmul2_rn(mx, make_float2(fz, fz)),
                                     __fmul2_rn(mxy, make_float2(fz, fz))};
                const int home = k / kBundleX;   // upper row -> slot 0, lower row -> slot 1
                const int other = 1 - home;
                // two paths, not three: a miss flushes and clears the home
                // slot, then shares the home slot's add
                if (pc[other] == cell && pc[home] != cell) {
#pragma unroll
                    for (int h = 0; h < kSlots; ++h)
                        if (h == other)
#pragma unroll
                            for (int e = 0; e < 4; ++e) p[h][e] = __fadd2_rn(p[h][e], w[e]);
                } else {
#pragma unroll
                    for (int h = 0; h < kSlots; ++h) {
                        if (h != home) continue;
                        if (pc[h] != cell) {
                            if (pc[h] >= 0) flush_record(rec, pc[h], p[h], ws.rec_stride);
                            pc[h] = cell;
#pragma unroll
                            for (int e = 0; e < 4; ++e) p[h][e] = make_float2(0.0f, 0.0f);
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) p[h][e] = __fadd2_rn(p[h][e], w[e]);
                    }
                }
            }
        }
#pragma unroll
        for (int h = 0; h < kSlots; ++h)
            if (pc[h] >= 0) flush_record(rec, pc[h], p[h], ws.rec_stride);
    }
}

// Slab records for the sparse views (rays about a voxel apart or more).
// With a workspace those views leave the direct path for per-cell records,
// built one slab of cell layers at a time: a slab's records (at most
// kSlabRecordBytes) stay in the L2, which the whole record array (8 floats
// per cell, 4x the gradient volume) does not, so every update is an L2
// reduction and no record goes to DRAM between two views.  A warp walks 8 x
// 4 neighbouring rays, each over the samples whose cell lies in the slab,
// keeps the moments of its current cell pending and flushes them (two
// 16-byte vector reductions into one sector) when the cell changes.  A ray
// about a voxel per sample changes cell nearly every sample, and the record
// then costs 2 sector operations per sample where the direct path's faces
// cost 3.5 (measured on the 256^3 volume seen by 64 views of 200^2 with 256
// samples: 1.93 reduction sectors per sample).  Then the slab's records go
// into the gradient (moments to corner weights, as scatter_records) and are
// cleared for the next slab.
//
// One cooperative launch does every slab, its phases separated by a grid
// barrier, so that a call whose views are all dense pays one launch that
// returns at once (separate launches per slab and phase cost 0.13 ms on the
// 4-view 1024^2 workload, 2.7 us each).  Measured slab sizes on that 64-view
// workload (B200): 24 / 32 / 48 MiB, 7.08 / 6.82 / 6.74 ms (separate
// launches per slab: 16 / 24 / 32 / 48 / 64 / 96 MiB, 7.63 / 7.07 / 6.85 /
// 6.95 / 7.06 / 7.60 ms).
constexpr long long kSlabRecordBytes = 48ll << 20;
// Calls of fewer ray-samples than this (all views counted) send their sparse
// views to the direct path (launch_adjoint).
constexpr double kSlabMinSamples = 8.0 * (1 << 20);

// A barrier wait gives up after this long (the slowest legitimate phase of a
// huge call is far shorter); it then raises the abort word, so that every
// other CTA leaves at its next wait, and is counted in g_wait_timeouts.
constexpr unsigned long long kBarrierTimeoutNs = 20ull * 1000 * 1000 * 1000;
__device__ unsigned long long g_wait_timeouts;

// Sample indices i in [0, N) whose 32.32 coordinate q0 + i s lies in [z0, z1):
// an interval, since the coordinate is monotone in i.  Exact integer bounds,
// so consecutive slabs share no sample and miss none.
__device__ __forceinline__ void slab_range(long long q0, long long s, int N, long long z0,
                                           long long z1, int& i0, int& i1) {
    if (s == 0) {
        i0 = 0;
        i1 = (q0 >= z0 && q0 < z1) ? N : 0;
        return;
    }
    // first index at which the coordinate is >= z (s > 0) or < z (s < 0)
    auto first = [&](long long z) -> int {
        long long k;
        if (s > 0) k = q0 >= z ? 0 : (z - q0 + s - 1) / s;
        else k = q0 < z ? 0 : (q0 - z) / (-s) + 1;
        return (int)min(k, (long long)N);
    };
    if (s > 0) {
        i0 = first(z0);
        i1 = first(z1);
    } else {
        i0 = first(z1);
        i1 = first(z0);
    }
}

// Records of one slab [cz0, cz1): slot s at rec + s * slab_stride, cell (i, j,
// k) at ((k - cz0) * (ny-1) + j) * (nx-1) + i.  Work items are 8 x 4 ray
// blocks of the sparse views, taken by the grid's warps in turn.
template <int MODE>
__device__ __forceinline__ void slab_records(const float* __restrict__ grad_out,
                                             const float* __restrict__ fwd_out, const Geom g,
                                             const Workspace ws, int cz0, int cz1,
                                             long long slab_stride) {
    const int lane = threadIdx.x & 31;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const long long gwarp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int bx = (g.W + kWarpW - 1) / kWarpW, by = (g.H + kWarpH - 1) / kWarpH;
    const long long per_view = (long long)bx * by, items = per_view * g.B;
    const int cr = g.nx - 1, cs = (g.nx - 1) * (g.ny - 1);
    const long long z0 = (long long)cz0 << 32, z1 = (long long)cz1 << 32;
    const long long slots = batch_slots(g);
    for (long long item = gwarp; item < items; item += nwarps) {
        // Every lane takes the same items; lanes without work in an item
        // wait here for the others, so that the warp's lanes do not drift
        // onto different items (without this wait: 16.0 against 9.6 ms).
        __syncwarp();
        const int b = (int)(item / per_view);
        const int t = (int)(item - (long long)b * per_view);
        const int wy = t / bx, wx = t - wy * bx;
        if (ws.flags[1 + b] != 0) continue;      // dense view: records_kernel's
        const BatchItem it = batch_item(g, b);
        if (!in_bounds(it.slot * slab_stride, slab_stride, slots * slab_stride)) continue;
        float* const rec = ws.rec + it.slot * slab_stride;
        const int c = wx * kWarpW + (lane % kWarpW), r = wy * kWarpH + (lane / kWarpW);
        if (r >= g.H || c >= g.W) continue;
        const size_t pix = ((size_t)b * g.H + r) * g.W + c;
        if (!in_bounds(pix, 1, (long long)g.B * g.H * g.W)) continue;
        float go = grad_out[pix];
        if (MODE == 1) go *= 1.0f - fwd_out[pix];
        Ray ray;
        if (go == 0.0f || !ray_setup(ws.views[b], g, (double)c, (double)r, 0.0, ray)) continue;
        int i0, i1;
        slab_range(ray.q0[2], ray.s[2], g.N, z0, z1, i0, i1);
        if (i0 >= i1) continue;
        const float scale = go * (g.density_factor * ray.dt);
        long long qx = ray.q0[0] + (long long)i0 * ray.s[0];
        long long qy = ray.q0[1] + (long long)i0 * ray.s[1];
        long long qz = ray.q0[2] + (long long)i0 * ray.s[2];
        int pc = -1;
        float2 p[4];
        for (int i = i0; i < i1; ++i) {
            const int cell = (fix_cell(qz) - cz0) * cs + fix_cell(qy) * cr + fix_cell(qx);
            const float fx = fix_frac(qx), fy = fix_frac(qy), fz = fix_frac(qz);
            qx += ray.s[0];
            qy += ray.s[1];
            qz += ray.s[2];
            const float2 mx = make_float2(scale, scale * fx);
            const float2 mxy = __fmul2_rn(mx, make_float2(fy, fy));
            const float2 w[4] = {mx, mxy, __fmul2_rn(mx, make_float2(fz, fz)),
                                 __fmul2_rn(mxy, make_float2(fz, fz))};
            if (cell != pc) {
                if (pc >= 0) flush_record(rec, pc, p, slab_stride);
                pc = cell;
#pragma unroll
                for (int e = 0; e < 4; ++e) p[e] = w[e];
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) p[e] = __fadd2_rn(p[e], w[e]);
            }
        }
        flush_record(rec, pc, p, slab_stride);
    }
}

// A slab's records into the gradient (as scatter_records: moments to corner
// weights, 8 coalesced atomic adds per cell), each record cleared after it is
// read so that the next slab starts from zeros.  A CTA takes whole x rows.
// Records are read and cleared in the L2 (.cg): the reductions wrote them
// there, and the next slab's reductions reuse the lines.
__device__ __forceinline__ void slab_scatter(float* __restrict__ rec, long long slab_stride,
                                             float* __restrict__ grad, const Geom g, int slots,
                                             int cz0, int cz1) {
    const int nx = g.nx, ny = g.ny;
    const int crow = nx - 1, rows = (ny - 1) * (cz1 - cz0);   // cells per row, rows per slot
    const long long total = (long long)rows * slots;
    const long long nxy = (long long)nx * ny, nvox = nxy * g.nz;
    const float4 zero = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (long long row = blockIdx.x; row < total; row += gridDim.x) {
        const int slot = (int)(row / rows);
        const int rr = (int)(row - (long long)slot * rows);
        const int kk = rr / (ny - 1), j = rr - kk * (ny - 1);
        const int k = cz0 + kk;
        float4* __restrict__ r =
            reinterpret_cast<float4*>(rec + slot * slab_stride + (long long)rr * crow * 8);
        float* __restrict__ gr = grad + slot * nvox + k * nxy + (long long)j * nx;
        for (int i = threadIdx.x; i < crow; i += blockDim.x) {
            if (!in_bounds(((long long)rr * crow + i) * 8, 8, slab_stride)) continue;
            const float4 lo = __ldcg(r + 2 * i), hi = __ldcg(r + 2 * i + 1);
            __stcg(r + 2 * i, zero);
            __stcg(r + 2 * i + 1, zero);
            float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            moments_to_corner_weights(v);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const long long off = i + (e & 1) + ((e >> 1) & 1) * nx + (e >> 2) * nxy;
                if (v[e] != 0.0f && in_bounds(k * nxy + (long long)j * nx + off, 1, nvox))
                    red_add(gr + off, v[e]);
            }
        }
    }
}

// Every slab of the sparse views: clear the slab records, then per slab the
// records and the scatter, with a grid barrier after each phase.  Launched
// cooperatively (all CTAs resident); returns at once when no view is sparse.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 4)
slab_adjoint_kernel(const float* __restrict__ grad_out, const float* __restrict__ fwd_out,
                    float* __restrict__ grad, const Geom g, const Workspace ws, int layers,
                    long long slab_stride) {
    if ((ws.flags[0] & kSomeSparse) == 0) return;   // the same in every CTA
    const int slots = batch_slots(g);
    const long long n4 = slab_stride / 4 * slots;
    float4* const r4 = reinterpret_cast<float4*>(ws.rec);
    const float4 zero = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (long long m = (long long)blockIdx.x * blockDim.x + threadIdx.x; m < n4;
         m += (long long)gridDim.x * blockDim.x)
        __stcg(r4 + m, zero);
    unsigned epoch = 0;
    if (!grid_barrier(ws.bar, epoch, gridDim.x, kBarrierTimeoutNs, &g_wait_timeouts)) return;
    for (int cz0 = 0; cz0 < g.nz - 1; cz0 += layers) {
        const int cz1 = min(cz0 + layers, g.nz - 1);
        slab_records<MODE>(grad_out, fwd_out, g, ws, cz0, cz1, slab_stride);
        if (!grid_barrier(ws.bar, epoch, gridDim.x, kBarrierTimeoutNs, &g_wait_timeouts)) return;
        slab_scatter(ws.rec, slab_stride, grad, g, slots, cz0, cz1);
        if (!grid_barrier(ws.bar, epoch, gridDim.x, kBarrierTimeoutNs, &g_wait_timeouts)) return;
    }
}

// Volume gradient of the alpha-composited image (front to back, the over
// operator; see march_alpha in drr_forward.cu): C = sum_i T_i a_i mu_i with
// a_i = 1 - exp(-s mu_i), s = density_factor * dt, T_{i+1} = T_i (1 - a_i).
// dC/dmu_i has a closed form in quantities known when sample i is reached
// front to back:
//   dC/dmu_i = T_i (s (1 - a_i) mu_i + a_i) - s (C - C_i),
// C_i = sum_{k <= i} T_k a_k mu_k, C the ray's image value (fwd_out) -- the
// later samples see sample i's absorption through T.  The kernel reads the
// volume (linear, corner or quad layout: the forward's own sample values),
// walks each ray once, front to back (no phases: T is sequential), and
// scatters grad_out * dC/dmu_i * w_corner through the pending 2 x 2 x 2
// block of the direct path into the fp32 linear gradient volume.
template <typename T, int LAYOUT, bool BATCH>
__global__ void __launch_bounds__(kThreads)
alpha_adjoint_kernel(const T* __restrict__ vol_base, const float* __restrict__ Rt,
                     const float* __restrict__ grad_out, const float* __restrict__ fwd_out,
                     float* __restrict__ grad, const Geom g, int grad_row, int grad_slice,
                     const int* __restrict__ flags) {
    __shared__ View sv;
    const int b = blockIdx.z;                    // output image (view x channel)
    if (flags && flags[1 + b]) return;           // dense view: alpha_records_kernel's
    // batches (a separate instantiation, so that single-volume calls carry
    // none of its registers): the image's pose and volume-channel
    const T* __restrict__ vol = vol_base;
    int pose = b;
    if constexpr (BATCH) {
        const BatchItem it = batch_item(g, b);
        const long long slots = batch_slots(g), nv = (long long)g.nx * g.ny * g.nz;
        if (!in_bounds(it.slot * g.vstride, g.vstride, slots * g.vstride) ||
            !in_bounds(it.slot * nv, nv, slots * nv))
            return;
        vol += it.slot * g.vstride;
        grad += it.slot * nv;
        pose = it.pose;
    }
    if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)pose, g, sv);
    __syncthreads();
    int r, c;
    tile_pixel(r, c);
    if (r >= g.H || c >= g.W) return;
    const size_t pix = ((size_t)b * g.H + r) * g.W + c;
    if (!in_bounds(pix, 1, (long long)g.B * g.H * g.W)) return;
    const float go = grad_out[pix];
    Ray ray;
    if (go == 0.0f || !ray_setup(sv, g, (double)c, (double)r, 0.0, ray)) return;
    const float Cray = fwd_out[pix];
    const float s = g.density_factor * ray.dt;
    const int st[3] = {1, grad_row, grad_slice};
    const long long nvox = (long long)g.nx * g.ny * g.nz;
    long long qx = ray.q0[0], qy = ray.q0[1], qz = ray.q0[2];
    int cell[3] = {fix_cell(qx), fix_cell(qy), fix_cell(qz)};
    float a8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a8[k] = 0.0f;
    float Ci = 0.0f, Tr = 1.0f;
    for (int i = 0; i < g.N; ++i) {
        const int cx = fix_cell(qx), cy = fix_cell(qy), cz = fix_cell(qz);
        const float fx = fix_frac(qx), fy = fix_frac(qy), fz = fix_frac(qz);
        // the forward's sample value, bit for bit
        const int at = cell_index<LAYOUT>(g, cx, cy, cz);
        const float mu =
            !in_bounds(sample_offset<LAYOUT>(at), sample_extent<LAYOUT>(g), g.vstride) ? 0.0f
            : LAYOUT == 4 ? sample_brick(vol + at, fx, fy, fz)
            : LAYOUT == 2 ? sample_corners(vol + (size_t)at * 8, fx, fy, fz)
            : LAYOUT == 3 ? sample_quads(vol + (size_t)at * 4, g.slice, fx, fy, fz)
                          : trilinear_at(vol + at, g.row, g.slice, fx, fy, fz);
        const float a = opacity<T>(s * mu);
        Ci = fmaf(Tr * a, mu, Ci);
        const float dmu = Tr * fmaf(s * (1.0f - a), mu, a) - s * (Cray - Ci);
        Tr *= 1.0f - a;
        const float scale = go * dmu;
        const int dx = cx - cell[0], dy = cy - cell[1], dz = cz - cell[2];
        if (dx < -1 || dx > 1 || dy < -1 || dy > 1 || dz < -1 || dz > 1) {
            flush_block(grad, st, cell, a8, nvox);
#pragma unroll
            for (int k = 0; k < 8; ++k) a8[k] = 0.0f;
            cell[0] = cx;
            cell[1] = cy;
            cell[2] = cz;
        } else {
            slide<0>(dx, grad, st, cell, a8, nvox);
            slide<1>(dy, grad, st, cell, a8, nvox);
            slide<2>(dz, grad, st, cell, a8, nvox);
        }
        const float wz1 = scale * fz, wz0 = scale * (1.0f - fz);
        const float w00 = wz0 * (1.0f - fy), w01 = wz0 * fy;
        const float w10 = wz1 * (1.0f - fy), w11 = wz1 * fy;
        const float gx = 1.0f - fx;
        a8[0] += w00 * gx;
        a8[1] += w00 * fx;
        a8[2] += w01 * gx;
        a8[3] += w01 * fx;
        a8[4] += w10 * gx;
        a8[5] += w10 * fx;
        a8[6] += w11 * gx;
        a8[7] += w11 * fx;
        qx += ray.s[0];
        qy += ray.s[1];
        qz += ray.s[2];
    }
    flush_block(grad, st, cell, a8, nvox);
}

// Record path of the alpha gradient for the views the plan marked dense: the
// per-sample factor of alpha_adjoint_kernel, accumulated like records_kernel.
// Each thread owns a 2 x 2 bundle of neighbouring rays (a CTA a 32 x 32 pixel
// tile) and two record slots, home to the bundle's rows; every ray carries
// its own T and C_i front to back, so there are no phases.  2 x 2 rather
// than 3 x 2: each ray also holds its sampling and compositing state.
// Measured on the 256^3 bf16 volume seen by 4 views of 1024^2, 512 samples:
// 12.0 ms against 31.4 for the direct path; 3 x 2 bundles 13.4 ms (spills
// at 128 registers) or 19.6 ms (148 registers, 1 CTA per SM); packed fp32x2
// weights 12.1 ms.  The records hold moments, as records_kernel's, turned
// into weights by scatter_records (11.13 against 11.53 ms with weight
// records and a voxel-centric gather pass).
constexpr int kAlphaBundle = 2;                          // rays per bundle, across and down
constexpr int kAlphaTile = 16 * kAlphaBundle;            // 32 x 32 pixels per CTA

template <typename T, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 2)
alpha_records_kernel(const T* __restrict__ vol_base, const float* __restrict__ Rt,
                     const float* __restrict__ grad_out, const float* __restrict__ fwd_out,
                     const Geom g, const Workspace ws) {
    constexpr int kRays = kAlphaBundle * kAlphaBundle;
    __shared__ View sv;
    const int b = blockIdx.z;
    if (ws.flags[1 + b] == 0) return;            // sparse view: alpha_adjoint_kernel's
    const BatchItem it = batch_item(g, b);
    const long long slots = batch_slots(g);
    if (!in_bounds(it.slot * g.vstride, g.vstride, slots * g.vstride) ||
        !in_bounds(it.slot * ws.rec_stride, ws.rec_stride, slots * ws.rec_stride))
        return;
    const T* __restrict__ vol = vol_base + it.slot * g.vstride;
    float* const rec = ws.rec + it.slot * ws.rec_stride;   // this volume-channel's records
    if (threadIdx.x == 0) view_setup(Rt + 12 * (size_t)it.pose, g, sv);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int px = (warp & 1) * 8 + (lane & 7), py = (warp >> 1) * 4 + (lane >> 3);
    const int c0 = blockIdx.x * kAlphaTile + px * kAlphaBundle;
    const int r0 = blockIdx.y * kAlphaTile + py * kAlphaBundle;

    bool act[kRays];
    float go[kRays], sa[kRays], Cray[kRays], Ci[kRays], Tr[kRays];
    long long q[kRays][3], s[kRays][3];
#pragma unroll
    for (int k = 0; k < kRays; ++k) {
        const int c = c0 + (k % kAlphaBundle), r = r0 + (k / kAlphaBundle);
        act[k] = false;
        go[k] = sa[k] = Cray[k] = Ci[k] = 0.0f;
        Tr[k] = 1.0f;
#pragma unroll
        for (int a = 0; a < 3; ++a) q[k][a] = s[k][a] = 0;
        if (r >= g.H || c >= g.W) continue;
        const size_t pix = ((size_t)b * g.H + r) * g.W + c;
        if (!in_bounds(pix, 1, (long long)g.B * g.H * g.W)) continue;
        go[k] = grad_out[pix];
        Ray ray;
        if (go[k] == 0.0f || !ray_setup(sv, g, (double)c, (double)r, 0.0, ray)) continue;
        act[k] = true;
        Cray[k] = fwd_out[pix];
        sa[k] = g.density_factor * ray.dt;
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            s[k][a] = ray.s[a];
            q[k][a] = ray.q0[a];
        }
    }
    // cells stay in [0, n-2] per axis (lim as for the linear layout), inside the records
    const int cr = g.nx - 1, cs = (g.nx - 1) * (g.ny - 1);
    float2 p[kSlots][4];
    int pc[kSlots];
#pragma unroll
    for (int h = 0; h < kSlots; ++h) pc[h] = -1;
    for (int i = 0; i < g.N; ++i) {
#pragma unroll
        for (int k = 0; k < kRays; ++k) {
            if (!act[k]) continue;
            const int cx = fix_cell(q[k][0]), cy = fix_cell(q[k][1]), cz = fix_cell(q[k][2]);
            const float fx = fix_frac(q[k][0]), fy = fix_frac(q[k][1]), fz = fix_frac(q[k][2]);
#pragma unroll
            for (int a = 0; a < 3; ++a) q[k][a] += s[k][a];
            // the forward's sample value, bit for bit
            const int at = cell_index<LAYOUT>(g, cx, cy, cz);
            const float mu =
                !in_bounds(sample_offset<LAYOUT>(at), sample_extent<LAYOUT>(g), g.vstride) ? 0.0f
                : LAYOUT == 4 ? sample_brick(vol + at, fx, fy, fz)
                : LAYOUT == 2 ? sample_corners(vol + (size_t)at * 8, fx, fy, fz)
                : LAYOUT == 3 ? sample_quads(vol + (size_t)at * 4, g.slice, fx, fy, fz)
                              : trilinear_at(vol + at, g.row, g.slice, fx, fy, fz);
            const float a = opacity<T>(sa[k] * mu);
            Ci[k] = fmaf(Tr[k] * a, mu, Ci[k]);
            const float dmu = Tr[k] * fmaf(sa[k] * (1.0f - a), mu, a) - sa[k] * (Cray[k] - Ci[k]);
            Tr[k] *= 1.0f - a;
            const float scale = go[k] * dmu;
            const int cell = cz * cs + cy * cr + cx;
            // the sample's 8 moments scale fx^a fy^b fz^c, as records_kernel
            const float2 mx = make_float2(scale, scale * fx);
            const float2 mxy = __fmul2_rn(mx, make_float2(fy, fy));
            const float2 w[4] = {mx, mxy, __fmul2_rn(mx, make_float2(fz, fz)),
                                 __fmul2_rn(mxy, make_float2(fz, fz))};
            const int home = k / kAlphaBundle, other = 1 - home;
            if (pc[other] == cell && pc[home] != cell) {
#pragma unroll
                for (int h = 0; h < kSlots; ++h)
                    if (h == other)
#pragma unroll
                        for (int e = 0; e < 4; ++e) p[h][e] = __fadd2_rn(p[h][e], w[e]);
            } else {
#pragma unroll
                for (int h = 0; h < kSlots; ++h) {
                    if (h != home) continue;
                    if (pc[h] != cell) {
                        if (pc[h] >= 0) flush_record(rec, pc[h], p[h], ws.rec_stride);
                        pc[h] = cell;
#pragma unroll
                        for (int e = 0; e < 4; ++e) p[h][e] = make_float2(0.0f, 0.0f);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) p[h][e] = __fadd2_rn(p[h][e], w[e]);
                }
            }
        }
    }
#pragma unroll
    for (int h = 0; h < kSlots; ++h)
        if (pc[h] >= 0) flush_record(rec, pc[h], p[h], ws.rec_stride);
}

}  // namespace

size_t adjoint_workspace_header(int B) { return header_layout(B).rec; }

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};
}  // namespace

// Device address of the built-in scratch on the current device, looked up
// once per device with that device current (the first call on a device does
// it; that call should come before any stream capture).  The cache holds for
// the life of the process: a cudaDeviceReset in between leaves it stale.
cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, noalloc_scratch_bytes);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}

DRR_BOUNDS_READER(bounds_word_adjoint)

cudaError_t wait_timeouts(unsigned long long* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_wait_timeouts, sizeof(*out));
    if (e != cudaSuccess) return e;
    const unsigned long long zero = 0ull;
    return cudaMemcpyToSymbol(g_wait_timeouts, &zero, sizeof(zero));
}

size_t adjoint_workspace_bytes(int nx, int ny, int nz, int B, int slots) {
    return adjoint_workspace_header(B) +
           (size_t)(nx - 1) * (ny - 1) * (nz - 1) * 8 * sizeof(float) * (size_t)slots;
}

namespace {

// The workspace's parts (header_layout) for B output images, and the plan
// launch that fills its header.
Workspace workspace_parts(void* workspace, const Geom& g) {
    Workspace ws{};
    ws.phase_shift = 4;
    if (!workspace) return ws;
    char* const base = static_cast<char*>(workspace);
    const HeaderLayout h = header_layout(g.B);
    ws.flags = static_cast<int*>(workspace);
    ws.bar = reinterpret_cast<unsigned*>(base + h.bar);
    ws.views = reinterpret_cast<const View*>(base + h.views);
    ws.rec = reinterpret_cast<float*>(base + h.rec);
    ws.rec_stride = (long long)(g.nx - 1) * (g.ny - 1) * (g.nz - 1) * 8;
    return ws;
}

void launch_plan(const Workspace& ws, const float* Rt, const Geom& g, cudaStream_t stream) {
    plan_views<<<1, 256, 0, stream>>>(Rt, g, ws.flags, const_cast<View*>(ws.views), ws.bar);
}

// The sparse views' slab pass: one cooperative launch, as many CTAs as fit
// on the device at once.
cudaError_t launch_slabs(const Workspace& ws, const Geom& g, int mode, const float* grad_out,
                         const float* fwd_out, float* grad_vol, cudaStream_t stream) {
    const int slots = batch_slots(g);
    const long long layer = (long long)(g.nx - 1) * (g.ny - 1) * 8;   // floats per cell layer
    int layers = (int)std::max(1LL, std::min((long long)(g.nz - 1),
                                             kSlabRecordBytes / (layer * 4 * slots)));
    long long slab_stride = layer * layers;
    const void* fn = mode == 1 ? (const void*)slab_adjoint_kernel<1>
                               : (const void*)slab_adjoint_kernel<0>;
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorLaunchOutOfResources;
    Workspace w = ws;
    Geom gg = g;
    void* args[] = {(void*)&grad_out, (void*)&fwd_out, (void*)&grad_vol, (void*)&gg, (void*)&w,
                    (void*)&layers, (void*)&slab_stride};
    return cudaLaunchCooperativeKernel(fn, dim3(sms * per_sm), dim3(kThreads), args, 0, stream);
}

}  // namespace

cudaError_t launch_adjoint(const Geom& g, const float* Rt, int mode, const float* grad_out,
                           const float* fwd_out, float* grad_vol, void* workspace,
                           cudaStream_t stream) {
    if (!workspace) {
        const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
        const Workspace none = workspace_parts(nullptr, g);
        if (mode == 1)
            adjoint_kernel<1><<<grid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, grad_vol, g,
                                                             none);
        else
            adjoint_kernel<0><<<grid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, grad_vol, g,
                                                             none);
        return cudaGetLastError();
    }
    Workspace ws = workspace_parts(workspace, g);
    const int slots = batch_slots(g);
    const int fill_grid = 148 * 8;
    // Phases over the whole ray keep warps that cover neighbouring rays off
    // the same records at the same time; over a record array many times the
    // L2 they also keep every record of the CTAs' beams live at once.
    // Beyond 1 GiB of records they span the first quarter of the ray instead
    // (B200: 4.3 GB of records for 2 views of 2048^2, 10.79 -> 10.48 ms; 530
    // MB for 4 views of 1024^2, the whole ray stays best: 6.00 against 6.03
    // ms).
    const double rec_bytes = (double)ws.rec_stride * 4.0 * slots;
    ws.phase_shift = rec_bytes > 1073741824.0 ? 6 : 4;
    launch_plan(ws, Rt, g, stream);
    zero_records<<<fill_grid, 256, 0, stream>>>(ws.flags, kSomeDense,
                                                reinterpret_cast<float4*>(ws.rec),
                                                ws.rec_stride / 4 * slots);
    const dim3 rgrid((g.W + kRecTileW - 1) / kRecTileW, (g.H + kRecTileH - 1) / kRecTileH, g.B);
    if (mode == 1)
        records_kernel<1><<<rgrid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, g, ws);
    else
        records_kernel<0><<<rgrid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, g, ws);
    scatter_records<<<fill_grid, 256, 0, stream>>>(ws.flags, ws.rec, ws.rec_stride, grad_vol, g.nx,
                                                   g.ny, g.nz, slots);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // The sparse views: slab by slab, in the (now scattered) record area; a
    // small call takes the direct path instead, where the slab pass's fixed
    // cost (clearing a slab, two grid barriers per slab: ~60 us) outweighs
    // its saving (~8 ps per ray-sample; 64^3 volume, one 64^2 view, 64
    // samples: 0.105 ms with the slab pass, 0.044 ms without).
    if ((double)g.B * g.H * g.W * g.N < kSlabMinSamples) {
        const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
        if (mode == 1)
            adjoint_kernel<1><<<grid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, grad_vol, g, ws);
        else
            adjoint_kernel<0><<<grid, kThreads, 0, stream>>>(Rt, grad_out, fwd_out, grad_vol, g, ws);
        return cudaGetLastError();
    }
    return launch_slabs(ws, g, mode, grad_out, fwd_out, grad_vol, stream);
}

template <typename T, int LAYOUT>
void alpha_kernels(const void* vol, const Geom& g, const float* Rt, const float* grad_out,
                   const float* fwd_out, float* grad_vol, const Workspace& ws,
                   cudaStream_t stream) {
    const T* v = static_cast<const T*>(vol);
    const dim3 grid((g.W + kTileW - 1) / kTileW, (g.H + kTileH - 1) / kTileH, g.B);
    if (g.C != 1 || g.broadcast || g.views_per_vol != g.B)
        alpha_adjoint_kernel<T, LAYOUT, true><<<grid, kThreads, 0, stream>>>(
            v, Rt, grad_out, fwd_out, grad_vol, g, g.nx, g.nx * g.ny, ws.flags);
    else
        alpha_adjoint_kernel<T, LAYOUT, false><<<grid, kThreads, 0, stream>>>(
            v, Rt, grad_out, fwd_out, grad_vol, g, g.nx, g.nx * g.ny, ws.flags);
    if (ws.flags) {
        const dim3 rgrid((g.W + kAlphaTile - 1) / kAlphaTile, (g.H + kAlphaTile - 1) / kAlphaTile,
                         g.B);
        alpha_records_kernel<T, LAYOUT><<<rgrid, kThreads, 0, stream>>>(v, Rt, grad_out, fwd_out,
                                                                         g, ws);
    }
}

cudaError_t launch_alpha_adjoint(const void* vol, int dtype, int layout, const Geom& g,
                                 const float* Rt, const float* grad_out, const float* fwd_out,
                                 float* grad_vol, void* workspace, cudaStream_t stream) {
    const Workspace ws = workspace_parts(workspace, g);
    const int fill_grid = 148 * 8;
    const int slots = batch_slots(g);
    if (workspace) {
        launch_plan(ws, Rt, g, stream);
        zero_records<<<fill_grid, 256, 0, stream>>>(ws.flags, kSomeDense,
                                                    reinterpret_cast<float4*>(ws.rec),
                                                    ws.rec_stride / 4 * slots);
    }
    if (dtype == 0) {
        if (layout == 4) alpha_kernels<float, 4>(vol, g, Rt, grad_out, fwd_out, grad_vol, ws, stream);
        else if (layout == 3) alpha_kernels<float, 3>(vol, g, Rt, grad_out, fwd_out, grad_vol, ws, stream);
        else if (layout == 2) alpha_kernels<float, 2>(vol, g, Rt, grad_out, fwd_out, grad_vol, ws, stream);
        else alpha_kernels<float, 0>(vol, g, Rt, grad_out, fwd_out, grad_vol, ws, stream);
    } else {
        if (layout == 4) alpha_kernels<uint16_t, 4>(vol, g, Rt, grad_out, fwd_out, grad_vol, ws, stream);
        else if (layout == 3) alpha_kernels<uint16_t, 3>(vol, g, Rt, grad_out, fwd_out, grad_vol, ws, stream);
        else if (layout == 2) alpha_kernels<uint16_t, 2>(vol, g, Rt, grad_out, fwd_out, grad_vol, ws, stream);
        else alpha_kernels<uint16_t, 0>(vol, g, Rt, grad_out, fwd_out, grad_vol, ws, stream);
    }
    if (workspace)
        scatter_records<<<fill_grid, 256, 0, stream>>>(ws.flags, ws.rec, ws.rec_stride, grad_vol,
                                                       g.nx, g.ny, g.nz, slots);
    return cudaGetLastError();
}

}  // namespace drr

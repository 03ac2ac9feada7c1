/*
 * drr_oracle.c -- fp64 CPU oracle of the cone-beam DRR ray-march.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, the smoke check in
 * __graft_entry__ and the cpu_baseline leg of bench.py may load this
 * library.  It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes, step by step, in the order of the method:
 *
 *  1. Camera ray (nanodrr page, introduction: Hartley-Zisserman pinhole
 *     x ~ K [R | t] X).  Pixel (row r, column c) has its centre at
 *     (u, v) = (c, r).  Solve K q = (u, v, 1) by back substitution (K is
 *     upper triangular), direction d = R^T q normalised to unit length in
 *     world mm, camera centre C = -R^T t.
 *  2. World -> IJK (flashdrr.rendering API docs, VolumeRaycaster.forward:
 *     the volume lives in IJK voxel space and an affine maps world to IJK;
 *     here the axis-aligned case x_world = origin + spacing * ijk, origin
 *     being the centre of voxel 0): C_ijk = (C - origin) / spacing,
 *     d_ijk = d / spacing, so a ray parameter t stays in world mm.
 *  3. Clip to the volume (flashdrr.rendering API docs,
 *     compute_clipping_distances: near/far from the volume bounds in IJK
 *     space), done per ray with the slab method on the box spanned by the
 *     voxel centres, [0, n-1] per axis.  A zero direction component is a
 *     miss if C lies outside that slab and no constraint otherwise.
 *     t0 = max(t_near, 0), t1 = t_far; t1 <= t0 is a miss (integral 0).
 *  4. N samples along each camera ray (VolumeRaycaster.__init__, parameter
 *     ray_samples), read as the midpoint rule: dt = (t1 - t0) / N,
 *     t_i = t0 + (i + 1/2) dt; each sample is a zero-padded trilinear
 *     interpolation of the volume (the grid_sample path of VolumeRaycaster)
 *     at C_ijk + t_i d_ijk; the samples are summed in order, in fp64.
 *  5. I = density_factor * dt * sum (VolumeRaycaster.__init__, parameter
 *     density_factor).  Output RAW: I; BEER_LAMBERT: 1 - exp(-I)
 *     (parameter use_beer_lambert), evaluated as -expm1(-I).
 *  6. Adjoint (TorchTomo page, "Discrete Adjoint and Learned Primal-Dual":
 *     the transpose satisfies <A x, y> = <x, A^T y>): the same loop, each
 *     sample scattering g * w_corner into the gradient volume, with
 *     g = grad_out * density_factor * dt, times exp(-I) in Beer-Lambert
 *     mode (the derivative of 1 - exp(-I)); I is the oracle's own forward.
 *  7. bf16 storage: round-to-nearest-even of the fp32 bit pattern to the
 *     upper 16 bits (the IEEE rounding rule, written out).
 *  9. Front-to-back alpha compositing, the over operator (flashdrr.rendering
 *     API docs, VolumeRaycaster.__init__: use_beer_lambert = False, with
 *     density_factor scaling the intensities before integration), read as
 *     the emission-absorption sum: sample i has opacity
 *     a_i = 1 - exp(-density_factor * mu_i * dt) and colour mu_i; with
 *     T_0 = 1 and T_{i+1} = T_i (1 - a_i) the image is C = sum T_i a_i mu_i,
 *     summed front (camera side) to back.  Its volume gradient is the
 *     reverse-mode derivative of that recurrence, accumulated back to front.
 * 10. Gaussian-Poisson surrogate (flashdrr.rendering API docs,
 *     VolumeRaycaster.apply_poisson): transmission T' = clamp(T + sqrt(T/i0) z,
 *     0, 1) with z ~ N(0, 1) given; here applied to a Beer-Lambert image
 *     1 - T (so T = 1 - image) and returning 1 - T'; its derivative with
 *     respect to the image is 1 + z / (2 sqrt(T i0)) where the clamp is
 *     inactive (0 < T + sqrt(T/i0) z < 1, T > 0), else 0.
 * 11. Cell-constant (Siddon) projector (diffct page, Features: project() and
 *     backproject() form an exact adjoint pair for the cell-constant Siddon
 *     model): voxel (i, j, k) is the cube [i - 1/2, i + 1/2] x ... in IJK with
 *     the constant value vol[k][j][i], and the ray's integral is the exact
 *     line integral of that piecewise-constant function: clip to the cells'
 *     box [-1/2, n - 1/2] per axis (t0 = max(t_near, 0) as before), split the
 *     chord at every plane x_a = m + 1/2 it crosses (the crossings sorted),
 *     and sum length (mm) x value of the cell holding each piece's midpoint,
 *     times density_factor.  The backprojection scatters the same lengths.
 *  8. Pose gradient (flashdrr.rendering API docs, VolumeRaycaster: rendering
 *     is differentiable with respect to the view matrices): dL/d[R|t], the
 *     12 entries of each view's world-to-camera matrix taken as free
 *     variables, L = sum over pixels of grad_out * image.  Chain rule
 *     through every step above: d = R^T q / |R^T q|, C = -R^T t, the IJK
 *     map, the clip (t0 and t1 move with the plane each one lies on; t0
 *     pinned at 0 has no derivative), the sample positions
 *     t_i = t0 + (i + 1/2)(t1 - t0)/N, the trilinear interpolant (its
 *     gradient inside the cell of each sample) and the factor dt.
 *
 * Rays are independent, so the forward may run rays on several threads;
 * every ray is still summed sequentially, so the result does not depend on
 * the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_RAW 0
#define ORACLE_BEER_LAMBERT 1
#define ORACLE_ALPHA 2

typedef struct {
    int64_t n[3];         /* nx, ny, nz; i is the fastest index */
    double spacing[3];    /* mm per voxel along i, j, k */
    double origin[3];     /* world mm of the centre of voxel (0, 0, 0) */
} grid_t;

static int make_grid(const int dims[3], const double spacing[3],
                     const double origin[3], grid_t *g) {
    for (int a = 0; a < 3; ++a) {
        if (dims[a] < 1 || !(spacing[a] > 0.0)) return -1;
        g->n[a] = dims[a];
        g->spacing[a] = spacing[a];
        g->origin[a] = origin[a];
    }
    return 0;
}

/* Back substitution of K q = (u, v, 1), K = [k0 k1 k2; 0 k4 k5; 0 0 k8]. */
static void back_substitute(const double K[9], double u, double v, double q[3]) {
    q[2] = 1.0 / K[8];
    q[1] = (v - K[5] * q[2]) / K[4];
    q[0] = (u - K[1] * q[1] - K[2] * q[2]) / K[0];
}

/* Step 1: ray of pixel centre (u, v) in world coordinates. */
static void camera_ray(const double K[9], const double Rt[12], double u, double v,
                       double C[3], double d[3]) {
    double q[3];
    back_substitute(K, u, v, q);
    double norm2 = 0.0;
    for (int a = 0; a < 3; ++a) {
        /* (R^T q)_a = sum_r R[r][a] q[r]; (R^T t)_a likewise */
        double da = 0.0, ca = 0.0;
        for (int r = 0; r < 3; ++r) {
            da += Rt[4 * r + a] * q[r];
            ca += Rt[4 * r + a] * Rt[4 * r + 3];
        }
        d[a] = da;
        C[a] = -ca;
        norm2 += da * da;
    }
    double inv = 1.0 / sqrt(norm2);
    for (int a = 0; a < 3; ++a) d[a] *= inv;
}

/* Steps 2-3: ray in IJK, clipped to the box [lo, lo + n - 1 + 2 pad] per
 * axis with lo = -pad (pad 0: the voxel centres; 1/2: the cells of the
 * cell-constant model); returns 1 on a hit. */
static int ray_in_box(const grid_t *g, const double K[9], const double Rt[12], double u,
                      double v, double pad, double Cijk[3], double dijk[3], double *t0,
                      double *t1) {
    double C[3], d[3];
    camera_ray(K, Rt, u, v, C, d);
    double t_near = -INFINITY, t_far = INFINITY;
    for (int a = 0; a < 3; ++a) {
        Cijk[a] = (C[a] - g->origin[a]) / g->spacing[a];
        dijk[a] = d[a] / g->spacing[a];
        double lo = 0.0 - pad, hi = (double)(g->n[a] - 1) + pad;
        if (dijk[a] == 0.0) {
            if (Cijk[a] < lo || Cijk[a] > hi) return 0;
            continue;
        }
        double tA = (lo - Cijk[a]) / dijk[a];
        double tB = (hi - Cijk[a]) / dijk[a];
        double tmin = tA < tB ? tA : tB;
        double tmax = tA < tB ? tB : tA;
        if (tmin > t_near) t_near = tmin;
        if (tmax < t_far) t_far = tmax;
    }
    *t0 = t_near > 0.0 ? t_near : 0.0;
    *t1 = t_far;
    return (*t1 > *t0) ? 1 : 0;
}

static int ray_in_volume(const grid_t *g, const double K[9], const double Rt[12], double u,
                         double v, double Cijk[3], double dijk[3], double *t0, double *t1) {
    return ray_in_box(g, K, Rt, u, v, 0.0, Cijk, dijk, t0, t1);
}

static double voxel(const float *vol, const grid_t *g, int64_t i, int64_t j, int64_t k) {
    if (i < 0 || j < 0 || k < 0 || i >= g->n[0] || j >= g->n[1] || k >= g->n[2]) return 0.0;
    return (double)vol[(k * g->n[1] + j) * g->n[0] + i];
}

/* Zero-padded trilinear interpolation at IJK point p. */
static double trilinear(const float *vol, const grid_t *g, const double p[3]) {
    double fl[3], f[3];
    int64_t i0[3];
    for (int a = 0; a < 3; ++a) {
        fl[a] = floor(p[a]);
        f[a] = p[a] - fl[a];
        i0[a] = (int64_t)fl[a];
    }
    double s = 0.0;
    for (int dk = 0; dk < 2; ++dk)
        for (int dj = 0; dj < 2; ++dj)
            for (int di = 0; di < 2; ++di) {
                double w = (di ? f[0] : 1.0 - f[0]) * (dj ? f[1] : 1.0 - f[1]) *
                           (dk ? f[2] : 1.0 - f[2]);
                s += w * voxel(vol, g, i0[0] + di, i0[1] + dj, i0[2] + dk);
            }
    return s;
}

/* Step 4: parameter of sample i, the midpoint of the i-th of N equal parts. */
static double sample_t(double t0, double dt, int i) { return t0 + ((double)i + 0.5) * dt; }

/* Steps 4-5 for one ray: returns the integral I (0 on a miss). */
static double ray_integral(const float *vol, const grid_t *g, const double K[9],
                           const double Rt[12], double u, double v, int n_samples,
                           double density_factor, double *dt_out) {
    double C[3], d[3], t0, t1;
    *dt_out = 0.0;
    if (!ray_in_volume(g, K, Rt, u, v, C, d, &t0, &t1)) return 0.0;
    double dt = (t1 - t0) / (double)n_samples;
    double sum = 0.0;
    for (int i = 0; i < n_samples; ++i) {
        double t = sample_t(t0, dt, i);
        double p[3] = {C[0] + t * d[0], C[1] + t * d[1], C[2] + t * d[2]};
        sum += trilinear(vol, g, p);
    }
    *dt_out = dt;
    return density_factor * dt * sum;
}

static double apply_mode(double I, int mode) {
    return mode == ORACLE_BEER_LAMBERT ? -expm1(-I) : I;
}

/* Step 9 for one ray: the front-to-back over operator (0 on a miss). */
static double ray_alpha(const float *vol, const grid_t *g, const double K[9],
                        const double Rt[12], double u, double v, int n_samples,
                        double density_factor) {
    double C[3], d[3], t0, t1;
    if (!ray_in_volume(g, K, Rt, u, v, C, d, &t0, &t1)) return 0.0;
    double dt = (t1 - t0) / (double)n_samples;
    double T = 1.0, out = 0.0;
    for (int i = 0; i < n_samples; ++i) {
        double t = sample_t(t0, dt, i);
        double p[3] = {C[0] + t * d[0], C[1] + t * d[1], C[2] + t * d[2]};
        double mu = trilinear(vol, g, p);
        double a = -expm1(-density_factor * mu * dt);
        out += T * a * mu;
        T *= 1.0 - a;
    }
    return out;
}

/* ------------------------------------------------------------------------ */
/* forward over a list of rays, threaded over contiguous chunks of rays      */

typedef struct {
    const float *vol;
    const grid_t *g;
    const double *K, *Rt;
    int H, W, n_samples, mode;
    double density_factor;
    const int64_t *ray_ids;   /* NULL: rays [begin, end) in order */
    int64_t begin, end;
    double *out;
} fwd_job_t;

static void *fwd_worker(void *arg) {
    fwd_job_t *job = (fwd_job_t *)arg;
    const int64_t hw = (int64_t)job->H * job->W;
    for (int64_t n = job->begin; n < job->end; ++n) {
        int64_t id = job->ray_ids ? job->ray_ids[n] : n;
        int64_t b = id / hw, rc = id % hw;
        double u = (double)(rc % job->W), v = (double)(rc / job->W);
        if (job->mode == ORACLE_ALPHA) {
            job->out[n] = ray_alpha(job->vol, job->g, job->K, job->Rt + 12 * b, u, v,
                                    job->n_samples, job->density_factor);
            continue;
        }
        double dt;
        double I = ray_integral(job->vol, job->g, job->K, job->Rt + 12 * b, u, v,
                                job->n_samples, job->density_factor, &dt);
        job->out[n] = apply_mode(I, job->mode);
    }
    return NULL;
}

static int run_forward(const float *vol, const grid_t *g, const double *K, const double *Rt,
                       int H, int W, int n_samples, double df, int mode,
                       const int64_t *ray_ids, int64_t n_rays, double *out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > n_rays) nthreads = n_rays > 0 ? (int)n_rays : 1;
    pthread_t tid[256];
    int running[256];
    fwd_job_t jobs[256];
    int64_t chunk = (n_rays + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        int64_t begin = t * chunk, end = (t + 1) * chunk;
        if (begin > n_rays) begin = n_rays;
        if (end > n_rays) end = n_rays;
        fwd_job_t j = {vol, g, K, Rt, H, W, n_samples, mode, df, ray_ids, begin, end, out};
        jobs[t] = j;
        running[t] = 0;
        if (begin >= end) continue;
        if (nthreads > 1 && pthread_create(&tid[t], NULL, fwd_worker, &jobs[t]) == 0)
            running[t] = 1;
        else
            fwd_worker(&jobs[t]);   /* one thread, or thread creation failed */
    }
    for (int t = 0; t < nthreads; ++t)
        if (running[t]) pthread_join(tid[t], NULL);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* exported API                                                              */

/* Full image: out[b][r][c], B*H*W doubles. Returns 0, or -1 on bad sizes. */
int oracle_render(const float *vol, const int dims[3], const double spacing[3],
                  const double origin[3], const double K[9], const double *Rt, int B,
                  int H, int W, int n_samples, double density_factor, int mode,
                  double *out, int nthreads) {
    grid_t g;
    if (make_grid(dims, spacing, origin, &g) || B < 0 || H < 0 || W < 0 || n_samples < 1)
        return -1;
    return run_forward(vol, &g, K, Rt, H, W, n_samples, density_factor, mode, NULL,
                       (int64_t)B * H * W, out, nthreads);
}

/* Selected rays, id = (b*H + r)*W + c; out[n] for ray_ids[n]. */
int oracle_render_rays(const float *vol, const int dims[3], const double spacing[3],
                       const double origin[3], const double K[9], const double *Rt, int B,
                       int H, int W, int n_samples, double density_factor, int mode,
                       const int64_t *ray_ids, int64_t n_rays, double *out, int nthreads) {
    grid_t g;
    if (make_grid(dims, spacing, origin, &g) || H < 1 || W < 1 || n_samples < 1) return -1;
    for (int64_t n = 0; n < n_rays; ++n)
        if (ray_ids[n] < 0 || ray_ids[n] >= (int64_t)B * H * W) return -1;
    return run_forward(vol, &g, K, Rt, H, W, n_samples, density_factor, mode, ray_ids,
                       n_rays, out, nthreads);
}

/* Ray geometry of one pixel: C_ijk, d_ijk (per mm), t0, t1. Returns hit flag. */
int oracle_ray(const int dims[3], const double spacing[3], const double origin[3],
               const double K[9], const double Rt[12], double u, double v,
               double Cijk[3], double dijk[3], double t01[2]) {
    grid_t g;
    if (make_grid(dims, spacing, origin, &g)) return -1;
    return ray_in_volume(&g, K, Rt, u, v, Cijk, dijk, &t01[0], &t01[1]);
}

/* Zero-padded trilinear interpolation at n points p[n][3] (IJK). */
int oracle_trilinear(const float *vol, const int dims[3], const double *p, int64_t n,
                     double *out) {
    grid_t g;
    const double one[3] = {1.0, 1.0, 1.0}, zero[3] = {0.0, 0.0, 0.0};
    if (make_grid(dims, one, zero, &g)) return -1;
    for (int64_t m = 0; m < n; ++m) out[m] = trilinear(vol, &g, p + 3 * m);
    return 0;
}

/* grad += go * w_corner * m at the 8 in-range corners of p. */
static void scatter(const grid_t *g, const double p[3], double m, double *grad) {
    double fl[3], f[3];
    int64_t i0[3];
    for (int a = 0; a < 3; ++a) {
        fl[a] = floor(p[a]);
        f[a] = p[a] - fl[a];
        i0[a] = (int64_t)fl[a];
    }
    for (int dk = 0; dk < 2; ++dk)
        for (int dj = 0; dj < 2; ++dj)
            for (int di = 0; di < 2; ++di) {
                int64_t ii = i0[0] + di, jj = i0[1] + dj, kk = i0[2] + dk;
                if (ii < 0 || jj < 0 || kk < 0 || ii >= g->n[0] || jj >= g->n[1] || kk >= g->n[2])
                    continue;
                double w = (di ? f[0] : 1.0 - f[0]) * (dj ? f[1] : 1.0 - f[1]) *
                           (dk ? f[2] : 1.0 - f[2]);
                grad[(kk * g->n[1] + jj) * g->n[0] + ii] += m * w;
            }
}

/* Step 9's volume gradient for one ray, by reverse-mode differentiation of
 * the recurrence C += T_i a_i mu_i, T_{i+1} = T_i (1 - a_i), with
 * a_i = 1 - exp(-s mu_i), s = density_factor * dt: going back to front with
 * Tbar = dC/dT_{i+1} (0 after the last sample),
 *   abar_i  = go T_i mu_i - Tbar T_i
 *   mubar_i = go T_i a_i + abar_i s (1 - a_i)
 *   Tbar    <- go a_i mu_i + Tbar (1 - a_i)   (= dC/dT_i)
 * and mubar_i scattered with the trilinear weights of sample i. */
static void alpha_ray_adjoint(const float *vol, const grid_t *g, const double C[3],
                              const double d[3], double t0, double dt, int n_samples,
                              double density_factor, double go, double *grad) {
    double *mu = (double *)malloc(sizeof(double) * 3 * (size_t)n_samples);
    if (!mu) return;
    double *a = mu + n_samples, *T = a + n_samples;
    const double s = density_factor * dt;
    double Tr = 1.0;
    for (int i = 0; i < n_samples; ++i) {
        double t = sample_t(t0, dt, i);
        double p[3] = {C[0] + t * d[0], C[1] + t * d[1], C[2] + t * d[2]};
        mu[i] = trilinear(vol, g, p);
        a[i] = -expm1(-s * mu[i]);
        T[i] = Tr;
        Tr *= 1.0 - a[i];
    }
    double Tbar = 0.0;
    for (int i = n_samples - 1; i >= 0; --i) {
        double abar = go * T[i] * mu[i] - Tbar * T[i];
        double mubar = go * T[i] * a[i] + abar * s * (1.0 - a[i]);
        Tbar = go * a[i] * mu[i] + Tbar * (1.0 - a[i]);
        double t = sample_t(t0, dt, i);
        double p[3] = {C[0] + t * d[0], C[1] + t * d[1], C[2] + t * d[2]};
        scatter(g, p, mubar, grad);
    }
    free(mu);
}

/* Adjoint of one view: grad[k][j][i] += sum over its rays and samples of
 * g * w_corner, accumulated in order. */
static void adjoint_view(const float *vol, const grid_t *g, const double K[9],
                         const double Rt[12], int H, int W, int n_samples,
                         double density_factor, int mode, const double *grad_out,
                         double *grad) {
    for (int r = 0; r < H; ++r)
        for (int c = 0; c < W; ++c) {
            double go = grad_out[(int64_t)r * W + c];
            double C[3], d[3], t0, t1;
            if (go == 0.0) continue;   /* contributes exactly nothing */
            if (!ray_in_volume(g, K, Rt, c, r, C, d, &t0, &t1)) continue;
            double dt = (t1 - t0) / (double)n_samples;
            if (mode == ORACLE_ALPHA) {
                alpha_ray_adjoint(vol, g, C, d, t0, dt, n_samples, density_factor, go, grad);
                continue;
            }
            double scale = go * density_factor * dt;
            if (mode == ORACLE_BEER_LAMBERT) {
                double dt2;
                double I = ray_integral(vol, g, K, Rt, c, r, n_samples, density_factor, &dt2);
                scale *= exp(-I);
            }
            for (int i = 0; i < n_samples; ++i) {
                double t = sample_t(t0, dt, i);
                double p[3] = {C[0] + t * d[0], C[1] + t * d[1], C[2] + t * d[2]};
                double fl[3], f[3];
                int64_t i0[3];
                for (int a = 0; a < 3; ++a) {
                    fl[a] = floor(p[a]);
                    f[a] = p[a] - fl[a];
                    i0[a] = (int64_t)fl[a];
                }
                for (int dk = 0; dk < 2; ++dk)
                    for (int dj = 0; dj < 2; ++dj)
                        for (int di = 0; di < 2; ++di) {
                            int64_t ii = i0[0] + di, jj = i0[1] + dj, kk = i0[2] + dk;
                            if (ii < 0 || jj < 0 || kk < 0 || ii >= g->n[0] || jj >= g->n[1] ||
                                kk >= g->n[2])
                                continue;
                            double w = (di ? f[0] : 1.0 - f[0]) * (dj ? f[1] : 1.0 - f[1]) *
                                       (dk ? f[2] : 1.0 - f[2]);
                            grad[(kk * g->n[1] + jj) * g->n[0] + ii] += scale * w;
                        }
            }
        }
}

typedef struct {
    const float *vol;
    const grid_t *g;
    const double *K, *Rt;
    int B, H, W, n_samples, mode, stride, first;
    double density_factor;
    const double *grad_out;
    double *grad;
} adj_job_t;

static void *adj_worker(void *arg) {
    adj_job_t *j = (adj_job_t *)arg;
    for (int b = j->first; b < j->B; b += j->stride)
        adjoint_view(j->vol, j->g, j->K, j->Rt + 12 * b, j->H, j->W, j->n_samples,
                     j->density_factor, j->mode, j->grad_out + (int64_t)b * j->H * j->W, j->grad);
    return NULL;
}

/* Adjoint: grad_vol[k][j][i] += A^T grad_out (times exp(-I) per ray in
 * Beer-Lambert mode, I from the oracle's own forward).  vol is read only in
 * Beer-Lambert mode and may be NULL in RAW.  With nthreads > 1, thread t
 * takes views t, t + nthreads, ... into a private fp64 buffer, and the
 * buffers are added to grad_vol in thread order, so the result depends only
 * on (inputs, nthreads). */
int oracle_adjoint(const float *vol, const int dims[3], const double spacing[3],
                   const double origin[3], const double K[9], const double *Rt, int B,
                   int H, int W, int n_samples, double density_factor, int mode,
                   const double *grad_out, double *grad_vol, int nthreads) {
    grid_t g;
    if (make_grid(dims, spacing, origin, &g) || B < 0 || H < 0 || W < 0 || n_samples < 1)
        return -1;
    if ((mode == ORACLE_BEER_LAMBERT || mode == ORACLE_ALPHA) && vol == NULL) return -1;
    if (nthreads > B) nthreads = B;
    if (nthreads > 64) nthreads = 64;
    if (nthreads < 1) nthreads = 1;
    const int64_t nvox = g.n[0] * g.n[1] * g.n[2];
    double *bufs[64];
    int got = 0;
    for (; got < nthreads && nthreads > 1; ++got) {
        bufs[got] = (double *)calloc((size_t)nvox, sizeof(double));
        if (!bufs[got]) break;
    }
    if (got < nthreads || nthreads == 1) {     /* one thread, straight into grad_vol */
        for (int t = 0; t < got; ++t) free(bufs[t]);
        adj_job_t j = {vol, &g, K, Rt, B, H, W, n_samples, mode, 1, 0, density_factor,
                       grad_out, grad_vol};
        adj_worker(&j);
        return 0;
    }
    pthread_t tid[64];
    int running[64];
    adj_job_t jobs[64];
    for (int t = 0; t < nthreads; ++t) {
        adj_job_t j = {vol, &g, K, Rt, B, H, W, n_samples, mode, nthreads, t, density_factor,
                       grad_out, bufs[t]};
        jobs[t] = j;
        running[t] = pthread_create(&tid[t], NULL, adj_worker, &jobs[t]) == 0;
        if (!running[t]) adj_worker(&jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        if (running[t]) pthread_join(tid[t], NULL);
    for (int t = 0; t < nthreads; ++t) {
        for (int64_t m = 0; m < nvox; ++m) grad_vol[m] += bufs[t][m];
        free(bufs[t]);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* pose gradient                                                             */

/* Gradient of the zero-padded trilinear interpolant at p, inside the cell
 * floor(p): d/dp_a of sum_corners w(f) v. */
static void trilinear_grad(const float *vol, const grid_t *g, const double p[3], double gr[3]) {
    double fl[3], f[3];
    int64_t i0[3];
    for (int a = 0; a < 3; ++a) {
        fl[a] = floor(p[a]);
        f[a] = p[a] - fl[a];
        i0[a] = (int64_t)fl[a];
        gr[a] = 0.0;
    }
    for (int dk = 0; dk < 2; ++dk)
        for (int dj = 0; dj < 2; ++dj)
            for (int di = 0; di < 2; ++di) {
                double v = voxel(vol, g, i0[0] + di, i0[1] + dj, i0[2] + dk);
                double wx = di ? f[0] : 1.0 - f[0], sx = di ? 1.0 : -1.0;
                double wy = dj ? f[1] : 1.0 - f[1], sy = dj ? 1.0 : -1.0;
                double wz = dk ? f[2] : 1.0 - f[2], sz = dk ? 1.0 : -1.0;
                gr[0] += sx * wy * wz * v;
                gr[1] += wx * sy * wz * v;
                gr[2] += wx * wy * sz * v;
            }
}

/* dI/d[R|t] of one ray, grad12[4r + c] for R[r][c] (c < 3) and t[r] (c = 3).
 * Returns the integral I (0 and a zero gradient on a miss).  In alpha mode
 * the derivative is of the composite C = sum_i T_i a_i mu_i instead (the
 * value returned is then C): each parameter's tangent is carried through the
 * front-to-back recurrence step by step -- dmu_i from the moved sample, ds =
 * density_factor * d(dt), da_i = (1 - a_i)(ds mu_i + s dmu_i), dC += dT_i a_i
 * mu_i + T_i da_i mu_i + T_i a_i dmu_i, dT_{i+1} = dT_i (1 - a_i) - T_i da_i. */
static double ray_pose_grad(const float *vol, const grid_t *g, const double K[9],
                            const double Rt[12], double u, double v, int n_samples,
                            double density_factor, int mode, double grad12[12]) {
    for (int m = 0; m < 12; ++m) grad12[m] = 0.0;
    double Cijk[3], dijk[3], t0, t1;
    if (!ray_in_volume(g, K, Rt, u, v, Cijk, dijk, &t0, &t1)) return 0.0;
    /* the camera ray again, with the pieces the derivatives need */
    double q[3], a[3], n2 = 0.0;
    back_substitute(K, u, v, q);
    for (int c = 0; c < 3; ++c) {
        a[c] = 0.0;
        for (int r = 0; r < 3; ++r) a[c] += Rt[4 * r + c] * q[r];
        n2 += a[c] * a[c];
    }
    const double nrm = sqrt(n2);
    double dw[3];
    for (int c = 0; c < 3; ++c) dw[c] = a[c] / nrm;
    /* which plane each end of the clip lies on: the axis that attains t_near
     * (the largest entry parameter) and t_far (the smallest exit one) */
    int ax0 = -1, ax1 = -1;
    double t_near = -INFINITY, t_far = INFINITY;
    for (int k = 0; k < 3; ++k) {
        if (dijk[k] == 0.0) continue;
        double tA = (0.0 - Cijk[k]) / dijk[k];
        double tB = ((double)(g->n[k] - 1) - Cijk[k]) / dijk[k];
        double tmin = tA < tB ? tA : tB, tmax = tA < tB ? tB : tA;
        if (tmin > t_near) { t_near = tmin; ax0 = k; }
        if (tmax < t_far) { t_far = tmax; ax1 = k; }
    }
    const int pinned0 = !(t_near > 0.0);   /* t0 = 0: the camera is inside the box */
    const double dt = (t1 - t0) / (double)n_samples;
    for (int m = 0; m < 12; ++m) {
        const int r = m / 4, c = m % 4;
        /* derivatives of the world camera centre and unit direction */
        double dC[3] = {0.0, 0.0, 0.0}, dd[3] = {0.0, 0.0, 0.0};
        if (c == 3) {
            /* C_w = -R^T t: dC_w[k]/dt[r] = -R[r][k]; d does not depend on t */
            for (int k = 0; k < 3; ++k) dC[k] = -Rt[4 * r + k];
        } else {
            /* dC_w[k]/dR[r][c] = -t[r] if k == c */
            dC[c] = -Rt[4 * r + 3];
            /* da/dR[r][c] = q[r] e_c; d(a/|a|) = (I - dw dw^T) da / |a| */
            for (int k = 0; k < 3; ++k)
                dd[k] = ((k == c ? 1.0 : 0.0) - dw[k] * dw[c]) * q[r] / nrm;
        }
        /* to IJK */
        for (int k = 0; k < 3; ++k) {
            dC[k] /= g->spacing[k];
            dd[k] /= g->spacing[k];
        }
        /* a clip plane x_k = P gives t = (P - C_k) / d_k */
        double dt0 = 0.0, dt1 = 0.0;
        if (!pinned0) dt0 = -(dC[ax0] + t0 * dd[ax0]) / dijk[ax0];
        dt1 = -(dC[ax1] + t1 * dd[ax1]) / dijk[ax1];
        const double ddt = (dt1 - dt0) / (double)n_samples;
        if (mode == ORACLE_ALPHA) {
            const double s = density_factor * dt, ds = density_factor * ddt;
            double T = 1.0, dT = 0.0, dCv = 0.0;
            for (int i = 0; i < n_samples; ++i) {
                const double ti = sample_t(t0, dt, i);
                const double dti = dt0 + ((double)i + 0.5) * ddt;
                double p[3], gr[3], dmu = 0.0;
                for (int k = 0; k < 3; ++k) p[k] = Cijk[k] + ti * dijk[k];
                const double mu = trilinear(vol, g, p);
                trilinear_grad(vol, g, p, gr);
                for (int k = 0; k < 3; ++k) dmu += gr[k] * (dC[k] + dti * dijk[k] + ti * dd[k]);
                const double a = -expm1(-s * mu);
                const double da = (1.0 - a) * (ds * mu + s * dmu);
                dCv += dT * a * mu + T * da * mu + T * a * dmu;
                dT = dT * (1.0 - a) - T * da;
                T *= 1.0 - a;
            }
            grad12[m] = dCv;
            continue;
        }
        double sum = 0.0, dsum = 0.0;
        for (int i = 0; i < n_samples; ++i) {
            const double ti = sample_t(t0, dt, i);
            const double dti = dt0 + ((double)i + 0.5) * ddt;
            double p[3], gr[3];
            for (int k = 0; k < 3; ++k) p[k] = Cijk[k] + ti * dijk[k];
            sum += trilinear(vol, g, p);
            trilinear_grad(vol, g, p, gr);
            for (int k = 0; k < 3; ++k) dsum += gr[k] * (dC[k] + dti * dijk[k] + ti * dd[k]);
        }
        grad12[m] = density_factor * (ddt * sum + dt * dsum);
    }
    if (mode == ORACLE_ALPHA) return ray_alpha(vol, g, K, Rt, u, v, n_samples, density_factor);
    double dt2;
    return ray_integral(vol, g, K, Rt, u, v, n_samples, density_factor, &dt2);
}

typedef struct {
    const float *vol;
    const grid_t *g;
    const double *K, *Rt;
    int B, H, W, n_samples, mode, stride, first;
    double density_factor;
    const double *grad_out;
    double *grad_Rt;
} pose_job_t;

static void *pose_worker(void *arg) {
    pose_job_t *j = (pose_job_t *)arg;
    for (int b = j->first; b < j->B; b += j->stride) {
        double acc[12] = {0.0};
        for (int r = 0; r < j->H; ++r)
            for (int c = 0; c < j->W; ++c) {
                double go = j->grad_out[((int64_t)b * j->H + r) * j->W + c];
                if (go == 0.0) continue;
                double g12[12];
                double I = ray_pose_grad(j->vol, j->g, j->K, j->Rt + 12 * b, c, r, j->n_samples,
                                         j->density_factor, j->mode, g12);
                /* Beer-Lambert: d(1 - exp(-I))/dI = exp(-I) */
                double w = go * (j->mode == ORACLE_BEER_LAMBERT ? exp(-I) : 1.0);
                for (int m = 0; m < 12; ++m) acc[m] += w * g12[m];
            }
        for (int m = 0; m < 12; ++m) j->grad_Rt[12 * b + m] += acc[m];
    }
    return NULL;
}

/* Pose gradient: grad_Rt[b][4r + c] += sum over the pixels of view b of
 * grad_out * d image / d Rt[b][r][c] (RAW, Beer-Lambert or alpha image).
 * Views run on up to nthreads threads;
 * each view is summed sequentially, so the result does not depend on the
 * thread count. */
int oracle_pose_grad(const float *vol, const int dims[3], const double spacing[3],
                     const double origin[3], const double K[9], const double *Rt, int B,
                     int H, int W, int n_samples, double density_factor, int mode,
                     const double *grad_out, double *grad_Rt, int nthreads) {
    grid_t g;
    if (make_grid(dims, spacing, origin, &g) || B < 0 || H < 0 || W < 0 || n_samples < 1)
        return -1;
    if (mode != ORACLE_RAW && mode != ORACLE_BEER_LAMBERT && mode != ORACLE_ALPHA) return -1;
    if (nthreads > B) nthreads = B;
    if (nthreads > 64) nthreads = 64;
    if (nthreads < 1) nthreads = 1;
    pthread_t tid[64];
    int running[64];
    pose_job_t jobs[64];
    for (int t = 0; t < nthreads; ++t) {
        pose_job_t j = {vol, &g, K, Rt, B, H, W, n_samples, mode, nthreads, t, density_factor,
                        grad_out, grad_Rt};
        jobs[t] = j;
        running[t] = nthreads > 1 && pthread_create(&tid[t], NULL, pose_worker, &jobs[t]) == 0;
        if (!running[t]) pose_worker(&jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        if (running[t]) pthread_join(tid[t], NULL);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* step 11: the cell-constant (Siddon) model                                 */

/* The ray clipped to the cells' box [-1/2, n - 1/2]; returns 1 on a hit. */
static int ray_in_cells(const grid_t *g, const double K[9], const double Rt[12], double u,
                        double v, double Cijk[3], double dijk[3], double *t0, double *t1) {
    return ray_in_box(g, K, Rt, u, v, 0.5, Cijk, dijk, t0, t1);
}

static int cmp_double(const void *a, const void *b) {
    double x = *(const double *)a, y = *(const double *)b;
    return x < y ? -1 : (x > y ? 1 : 0);
}

/* The pieces of one ray: ts[0] = t0 < ts[1] < ... < ts[n] = t1 at the plane
 * crossings; returns the number of pieces n (0 on a miss), ts malloc'ed. */
static int siddon_pieces(const grid_t *g, const double C[3], const double d[3], double t0,
                         double t1, double **ts_out) {
    int64_t cap = 2 + g->n[0] + g->n[1] + g->n[2];
    double *ts = (double *)malloc(sizeof(double) * (size_t)cap);
    if (!ts) return 0;
    int64_t m = 0;
    ts[m++] = t0;
    for (int a = 0; a < 3; ++a) {
        if (d[a] == 0.0) continue;
        for (int64_t k = 0; k + 1 < g->n[a]; ++k) {          /* interior planes x_a = k + 1/2 */
            double t = ((double)k + 0.5 - C[a]) / d[a];
            if (t > t0 && t < t1) ts[m++] = t;
        }
    }
    qsort(ts + 1, (size_t)(m - 1), sizeof(double), cmp_double);
    ts[m++] = t1;
    *ts_out = ts;
    return (int)(m - 1);
}

/* The cell holding IJK point p (nearest voxel centre), clamped into the box. */
static void siddon_cell(const grid_t *g, const double p[3], int64_t c[3]) {
    for (int a = 0; a < 3; ++a) {
        int64_t k = (int64_t)floor(p[a] + 0.5);
        if (k < 0) k = 0;
        if (k > g->n[a] - 1) k = g->n[a] - 1;
        c[a] = k;
    }
}

static double ray_siddon(const float *vol, const grid_t *g, const double K[9],
                         const double Rt[12], double u, double v, double density_factor) {
    double C[3], d[3], t0, t1, *ts = NULL;
    if (!ray_in_cells(g, K, Rt, u, v, C, d, &t0, &t1)) return 0.0;
    int n = siddon_pieces(g, C, d, t0, t1, &ts);
    double sum = 0.0;
    for (int s = 0; s < n; ++s) {
        double tm = 0.5 * (ts[s] + ts[s + 1]);
        double p[3] = {C[0] + tm * d[0], C[1] + tm * d[1], C[2] + tm * d[2]};
        int64_t c[3];
        siddon_cell(g, p, c);
        sum += (ts[s + 1] - ts[s]) * (double)vol[(c[2] * g->n[1] + c[1]) * g->n[0] + c[0]];
    }
    free(ts);
    return density_factor * sum;
}

/* Forward of the cell-constant model: out[b][r][c] (RAW or Beer-Lambert). */
int oracle_render_siddon(const float *vol, const int dims[3], const double spacing[3],
                         const double origin[3], const double K[9], const double *Rt, int B,
                         int H, int W, double density_factor, int mode, double *out) {
    grid_t g;
    if (make_grid(dims, spacing, origin, &g) || B < 0 || H < 0 || W < 0) return -1;
    if (mode != ORACLE_RAW && mode != ORACLE_BEER_LAMBERT) return -1;
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < H; ++r)
            for (int c = 0; c < W; ++c)
                out[((int64_t)b * H + r) * W + c] =
                    apply_mode(ray_siddon(vol, &g, K, Rt + 12 * b, c, r, density_factor), mode);
    return 0;
}

/* Backprojection of the cell-constant model: grad_vol += lengths x
 * grad_out x density_factor (x exp(-I) in Beer-Lambert, I from vol). */
int oracle_siddon_adjoint(const float *vol, const int dims[3], const double spacing[3],
                          const double origin[3], const double K[9], const double *Rt, int B,
                          int H, int W, double density_factor, int mode, const double *grad_out,
                          double *grad_vol) {
    grid_t g;
    if (make_grid(dims, spacing, origin, &g) || B < 0 || H < 0 || W < 0) return -1;
    if (mode != ORACLE_RAW && mode != ORACLE_BEER_LAMBERT) return -1;
    if (mode == ORACLE_BEER_LAMBERT && vol == NULL) return -1;
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < H; ++r)
            for (int c = 0; c < W; ++c) {
                double go = grad_out[((int64_t)b * H + r) * W + c];
                if (go == 0.0) continue;
                double C[3], d[3], t0, t1, *ts = NULL;
                if (!ray_in_cells(&g, K, Rt + 12 * b, c, r, C, d, &t0, &t1)) continue;
                double scale = go * density_factor;
                if (mode == ORACLE_BEER_LAMBERT)
                    scale *= exp(-ray_siddon(vol, &g, K, Rt + 12 * b, c, r, density_factor));
                int n = siddon_pieces(&g, C, d, t0, t1, &ts);
                for (int s = 0; s < n; ++s) {
                    double tm = 0.5 * (ts[s] + ts[s + 1]);
                    double p[3] = {C[0] + tm * d[0], C[1] + tm * d[1], C[2] + tm * d[2]};
                    int64_t cc[3];
                    siddon_cell(&g, p, cc);
                    grad_vol[(cc[2] * g.n[1] + cc[1]) * g.n[0] + cc[0]] += scale * (ts[s + 1] - ts[s]);
                }
                free(ts);
            }
    return 0;
}

/* Step 10: out[m] = 1 - clamp(T + sqrt(T / i0) z[m], 0, 1), T = 1 - image[m]. */
int oracle_poisson_noise(const double *image, const double *z, double i0, double *out,
                         int64_t n) {
    if (!(i0 > 0.0)) return -1;
    for (int64_t m = 0; m < n; ++m) {
        double T = 1.0 - image[m];
        double Tn = T > 0.0 ? T + sqrt(T / i0) * z[m] : T;
        if (Tn < 0.0) Tn = 0.0;
        if (Tn > 1.0) Tn = 1.0;
        out[m] = 1.0 - Tn;
    }
    return 0;
}

/* Its derivative: grad_image[m] = grad_out[m] * (1 + z / (2 sqrt(T i0))) where
 * 0 < T + sqrt(T / i0) z < 1 and T > 0, else 0. */
int oracle_poisson_noise_backward(const double *image, const double *z, double i0,
                                  const double *grad_out, double *grad_image, int64_t n) {
    if (!(i0 > 0.0)) return -1;
    for (int64_t m = 0; m < n; ++m) {
        double T = 1.0 - image[m];
        double slope = 0.0;
        if (T > 0.0) {
            double Tn = T + sqrt(T / i0) * z[m];
            if (Tn > 0.0 && Tn < 1.0) slope = 1.0 + z[m] / (2.0 * sqrt(T * i0));
        }
        grad_image[m] = grad_out[m] * slope;
    }
    return 0;
}

/* bf16 storage: round-to-nearest-even of each fp32 value to its upper 16
 * bits; NaN stays a (quiet) NaN. */
void oracle_round_bf16(const float *in, uint16_t *out, int64_t n) {
    for (int64_t m = 0; m < n; ++m) {
        uint32_t bits;
        memcpy(&bits, &in[m], 4);
        if ((bits & 0x7f800000u) == 0x7f800000u && (bits & 0x007fffffu)) {
            out[m] = (uint16_t)((bits >> 16) | 0x0040u);
            continue;
        }
        uint32_t lsb = (bits >> 16) & 1u;
        bits += 0x7fffu + lsb;
        out[m] = (uint16_t)(bits >> 16);
    }
}

/* Widen bf16 bit patterns back to fp32 values. */
void oracle_bf16_to_float(const uint16_t *in, float *out, int64_t n) {
    for (int64_t m = 0; m < n; ++m) {
        uint32_t bits = (uint32_t)in[m] << 16;
        memcpy(&out[m], &bits, 4);
    }
}

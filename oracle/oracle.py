"""ctypes binding of liboracle.so -- TEST INFRASTRUCTURE (see package doc).

All geometry is widened to fp64 here from whatever the caller passes (the
float32 arrays the GPU also sees); volumes are passed as float32.
"""
import ctypes
import os

import numpy as np

from .build import LIB, build

_lib = None
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_c = ctypes


def load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB):
        build()
    lib = ctypes.CDLL(LIB)
    lib.oracle_render.argtypes = [_f32p, _i32p, _f64p, _f64p, _f64p, _f64p, _c.c_int, _c.c_int,
                                  _c.c_int, _c.c_int, _c.c_double, _c.c_int, _f64p, _c.c_int]
    lib.oracle_render.restype = _c.c_int
    lib.oracle_render_rays.argtypes = [_f32p, _i32p, _f64p, _f64p, _f64p, _f64p, _c.c_int,
                                       _c.c_int, _c.c_int, _c.c_int, _c.c_double, _c.c_int,
                                       _i64p, _c.c_int64, _f64p, _c.c_int]
    lib.oracle_render_rays.restype = _c.c_int
    lib.oracle_ray.argtypes = [_i32p, _f64p, _f64p, _f64p, _f64p, _c.c_double, _c.c_double,
                               _f64p, _f64p, _f64p]
    lib.oracle_ray.restype = _c.c_int
    lib.oracle_trilinear.argtypes = [_f32p, _i32p, _f64p, _c.c_int64, _f64p]
    lib.oracle_trilinear.restype = _c.c_int
    lib.oracle_adjoint.argtypes = [_c.c_void_p, _i32p, _f64p, _f64p, _f64p, _f64p, _c.c_int,
                                   _c.c_int, _c.c_int, _c.c_int, _c.c_double, _c.c_int, _f64p,
                                   _f64p, _c.c_int]
    lib.oracle_adjoint.restype = _c.c_int
    lib.oracle_pose_grad.argtypes = [_f32p, _i32p, _f64p, _f64p, _f64p, _f64p, _c.c_int,
                                     _c.c_int, _c.c_int, _c.c_int, _c.c_double, _c.c_int,
                                     _f64p, _f64p, _c.c_int]
    lib.oracle_pose_grad.restype = _c.c_int
    lib.oracle_poisson_noise.argtypes = [_f64p, _f64p, _c.c_double, _f64p, _c.c_int64]
    lib.oracle_poisson_noise.restype = _c.c_int
    lib.oracle_poisson_noise_backward.argtypes = [_f64p, _f64p, _c.c_double, _f64p, _f64p,
                                                  _c.c_int64]
    lib.oracle_poisson_noise_backward.restype = _c.c_int
    lib.oracle_render_siddon.argtypes = [_f32p, _i32p, _f64p, _f64p, _f64p, _f64p, _c.c_int,
                                         _c.c_int, _c.c_int, _c.c_double, _c.c_int, _f64p]
    lib.oracle_render_siddon.restype = _c.c_int
    lib.oracle_siddon_adjoint.argtypes = [_c.c_void_p, _i32p, _f64p, _f64p, _f64p, _f64p,
                                          _c.c_int, _c.c_int, _c.c_int, _c.c_double, _c.c_int,
                                          _f64p, _f64p]
    lib.oracle_siddon_adjoint.restype = _c.c_int
    lib.oracle_round_bf16.argtypes = [_f32p, _u16p, _c.c_int64]
    lib.oracle_round_bf16.restype = None
    lib.oracle_bf16_to_float.argtypes = [_u16p, _f32p, _c.c_int64]
    lib.oracle_bf16_to_float.restype = None
    _lib = lib
    return lib


def _geom(dims, spacing, origin, K, Rt):
    dims = np.ascontiguousarray(dims, dtype=np.int32).reshape(3)
    spacing = np.ascontiguousarray(spacing, dtype=np.float64).reshape(3)
    origin = np.ascontiguousarray(origin, dtype=np.float64).reshape(3)
    K = np.ascontiguousarray(K, dtype=np.float64).reshape(9)
    Rt = np.ascontiguousarray(Rt, dtype=np.float64).reshape(-1, 12)
    return dims, spacing, origin, K, Rt


def _vol(vol, dims):
    v = np.ascontiguousarray(vol, dtype=np.float32)
    assert v.size == int(np.prod(dims)), "volume size does not match dims"
    return v.reshape(-1)


def render(vol, dims, spacing, origin, K, Rt, H, W, n_samples, density_factor, mode,
           nthreads=None):
    """Full image out[b][r][c] (float64)."""
    dims, spacing, origin, K, Rt = _geom(dims, spacing, origin, K, Rt)
    B = Rt.shape[0]
    out = np.zeros(B * H * W, dtype=np.float64)
    nt = nthreads or len(os.sched_getaffinity(0))
    rc = load().oracle_render(_vol(vol, dims), dims, spacing, origin, K, Rt.reshape(-1), B, H,
                              W, n_samples, density_factor, mode, out, nt)
    assert rc == 0, "oracle_render rejected its arguments"
    return out.reshape(B, H, W)


def render_rays(vol, dims, spacing, origin, K, Rt, H, W, n_samples, density_factor, mode,
                ray_ids, nthreads=None):
    """Selected rays (id = (b*H + r)*W + c), float64."""
    dims, spacing, origin, K, Rt = _geom(dims, spacing, origin, K, Rt)
    ids = np.ascontiguousarray(ray_ids, dtype=np.int64).reshape(-1)
    out = np.zeros(ids.size, dtype=np.float64)
    nt = nthreads or len(os.sched_getaffinity(0))
    rc = load().oracle_render_rays(_vol(vol, dims), dims, spacing, origin, K, Rt.reshape(-1),
                                   Rt.shape[0], H, W, n_samples, density_factor, mode, ids,
                                   ids.size, out, nt)
    assert rc == 0, "oracle_render_rays rejected its arguments"
    return out


def ray(dims, spacing, origin, K, Rt12, u, v):
    """(hit, C_ijk, d_ijk, t0, t1) of pixel centre (u, v) for one view."""
    dims, spacing, origin, K, Rt = _geom(dims, spacing, origin, K, Rt12)
    C = np.zeros(3)
    d = np.zeros(3)
    t01 = np.zeros(2)
    hit = load().oracle_ray(dims, spacing, origin, K, Rt.reshape(-1)[:12].copy(), float(u),
                            float(v), C, d, t01)
    assert hit in (0, 1)
    return bool(hit), C, d, t01[0], t01[1]


def trilinear(vol, dims, points):
    dims_a = np.ascontiguousarray(dims, dtype=np.int32).reshape(3)
    p = np.ascontiguousarray(points, dtype=np.float64).reshape(-1, 3)
    out = np.zeros(p.shape[0])
    rc = load().oracle_trilinear(_vol(vol, dims_a), dims_a, p.reshape(-1), p.shape[0], out)
    assert rc == 0
    return out


def adjoint(dims, spacing, origin, K, Rt, H, W, n_samples, density_factor, mode, grad_out,
            vol=None, nthreads=1):
    """grad_vol[k][j][i] (float64) = A^T grad_out (times exp(-I) in Beer-Lambert);
    in alpha mode (2) the volume gradient of the over-operator image, which
    needs vol."""
    dims, spacing, origin, K, Rt = _geom(dims, spacing, origin, K, Rt)
    B = Rt.shape[0]
    go = np.ascontiguousarray(grad_out, dtype=np.float64).reshape(-1)
    assert go.size == B * H * W
    grad = np.zeros(int(np.prod(dims)), dtype=np.float64)
    keep = None
    vptr = None
    if vol is not None:
        keep = _vol(vol, dims)
        vptr = keep.ctypes.data
    rc = load().oracle_adjoint(vptr, dims, spacing, origin, K, Rt.reshape(-1), B, H, W,
                               n_samples, density_factor, mode, go, grad, int(nthreads))
    assert rc == 0, "oracle_adjoint rejected its arguments"
    nx, ny, nz = (int(x) for x in dims)
    return grad.reshape(nz, ny, nx)


def pose_grad(vol, dims, spacing, origin, K, Rt, H, W, n_samples, density_factor, mode,
              grad_out, nthreads=1):
    """grad_Rt[b][r][c] (float64, B x 3 x 4) = sum over the pixels of view b of
    grad_out * d image / d Rt[b][r][c] (the 12 matrix entries taken as free
    variables; times exp(-I) in Beer-Lambert; of the composite in alpha
    mode)."""
    dims, spacing, origin, K, Rt = _geom(dims, spacing, origin, K, Rt)
    B = Rt.shape[0]
    go = np.ascontiguousarray(grad_out, dtype=np.float64).reshape(-1)
    assert go.size == B * H * W
    out = np.zeros(B * 12, dtype=np.float64)
    v = _vol(vol, dims)
    rc = load().oracle_pose_grad(v, dims, spacing, origin, K, Rt.reshape(-1), B, H, W,
                                 n_samples, density_factor, mode, go, out, int(nthreads))
    assert rc == 0, "oracle_pose_grad rejected its arguments"
    return out.reshape(B, 3, 4)


def poisson_noise(image, z, i0):
    """1 - clamp(T + sqrt(T / i0) z, 0, 1) with T = 1 - image (float64)."""
    img = np.ascontiguousarray(image, dtype=np.float64)
    zz = np.ascontiguousarray(z, dtype=np.float64)
    assert zz.shape == img.shape
    out = np.empty_like(img)
    rc = load().oracle_poisson_noise(img.reshape(-1), zz.reshape(-1), float(i0), out.reshape(-1),
                                     img.size)
    assert rc == 0, "oracle_poisson_noise rejected its arguments"
    return out


def poisson_noise_backward(image, z, i0, grad_out):
    """d/d(image) of poisson_noise, times grad_out (float64)."""
    img = np.ascontiguousarray(image, dtype=np.float64)
    zz = np.ascontiguousarray(z, dtype=np.float64)
    go = np.ascontiguousarray(grad_out, dtype=np.float64)
    assert zz.shape == img.shape == go.shape
    gi = np.empty_like(img)
    rc = load().oracle_poisson_noise_backward(img.reshape(-1), zz.reshape(-1), float(i0),
                                              go.reshape(-1), gi.reshape(-1), img.size)
    assert rc == 0, "oracle_poisson_noise_backward rejected its arguments"
    return gi


def render_siddon(vol, dims, spacing, origin, K, Rt, H, W, density_factor, mode):
    """Cell-constant (Siddon) image out[b][r][c] (float64), RAW or Beer-Lambert."""
    dims, spacing, origin, K, Rt = _geom(dims, spacing, origin, K, Rt)
    B = Rt.shape[0]
    out = np.zeros(B * H * W, dtype=np.float64)
    rc = load().oracle_render_siddon(_vol(vol, dims), dims, spacing, origin, K, Rt.reshape(-1),
                                     B, H, W, density_factor, mode, out)
    assert rc == 0, "oracle_render_siddon rejected its arguments"
    return out.reshape(B, H, W)


def siddon_adjoint(dims, spacing, origin, K, Rt, H, W, density_factor, mode, grad_out, vol=None):
    """Backprojection of the cell-constant model (float64 [nz][ny][nx])."""
    dims, spacing, origin, K, Rt = _geom(dims, spacing, origin, K, Rt)
    B = Rt.shape[0]
    go = np.ascontiguousarray(grad_out, dtype=np.float64).reshape(-1)
    assert go.size == B * H * W
    grad = np.zeros(int(np.prod(dims)), dtype=np.float64)
    keep = _vol(vol, dims) if vol is not None else None
    rc = load().oracle_siddon_adjoint(None if keep is None else keep.ctypes.data, dims, spacing,
                                      origin, K, Rt.reshape(-1), B, H, W, density_factor, mode,
                                      go, grad)
    assert rc == 0, "oracle_siddon_adjoint rejected its arguments"
    nx, ny, nz = (int(x) for x in dims)
    return grad.reshape(nz, ny, nx)


def batch_map(n_vols, channels, n_views):
    """The batch rule written out (VolumeRaycaster.forward: N = B *
    views_per_vol view matrices, N == 1 broadcast to B): a list of
    (output view n, pose row, volume v) for every output view."""
    if n_views == 1 and n_vols > 1:
        return [(n, 0, n) for n in range(n_vols)]
    assert n_views % n_vols == 0, "n_views must be 1 or a multiple of n_vols"
    per = n_views // n_vols
    return [(n, n, n // per) for n in range(n_views)]


def render_batched(vols, dims, spacing, origin, K, Rt, n_views, H, W, n_samples, density_factor,
                   mode, nthreads=None):
    """vols[v][ch] (n_vols x C x nz x ny x nx) -> out[n][ch][r][c] (float64),
    each image rendered alone by render()."""
    vols = np.asarray(vols)
    n_vols, C = vols.shape[0], vols.shape[1]
    Rt = np.asarray(Rt).reshape(-1, 12)
    items = batch_map(n_vols, C, n_views)
    out = np.zeros((len(items), C, H, W))
    for n, pose, v in items:
        for ch in range(C):
            out[n, ch] = render(vols[v, ch], dims, spacing, origin, K, Rt[pose:pose + 1], H, W,
                                n_samples, density_factor, mode, nthreads)[0]
    return out


def adjoint_batched(dims, spacing, origin, K, Rt, n_vols, n_views, H, W, n_samples,
                    density_factor, mode, grad_out, vols=None, nthreads=1):
    """grad_vols[v][ch] (float64) = sum over the images rendered from (v, ch)
    of their adjoints (adjoint() of each image alone)."""
    go = np.asarray(grad_out, np.float64)
    C = go.shape[1]
    Rt = np.asarray(Rt).reshape(-1, 12)
    nx, ny, nz = (int(x) for x in dims)
    grads = np.zeros((n_vols, C, nz, ny, nx))
    for n, pose, v in batch_map(n_vols, C, n_views):
        for ch in range(C):
            grads[v, ch] += adjoint(dims, spacing, origin, K, Rt[pose:pose + 1], H, W, n_samples,
                                    density_factor, mode, go[n, ch][None],
                                    vol=None if vols is None else np.asarray(vols)[v, ch],
                                    nthreads=nthreads)
    return grads


def pose_grad_batched(vols, dims, spacing, origin, K, Rt, n_views, H, W, n_samples,
                      density_factor, mode, grad_out, nthreads=1):
    """grad_Rt[p] (float64, n_views x 3 x 4) = sum over the images rendered
    with pose p of their pose gradients (pose_grad() of each image alone,
    with the volume-channel it was rendered from)."""
    vols = np.asarray(vols)
    n_vols, C = vols.shape[0], vols.shape[1]
    go = np.asarray(grad_out, np.float64)
    Rt = np.asarray(Rt).reshape(-1, 12)
    out = np.zeros((Rt.shape[0], 3, 4))
    for n, pose, v in batch_map(n_vols, C, n_views):
        for ch in range(C):
            out[pose] += pose_grad(vols[v, ch], dims, spacing, origin, K, Rt[pose:pose + 1], H, W,
                                   n_samples, density_factor, mode, go[n, ch][None],
                                   nthreads=nthreads)[0]
    return out


def round_bf16(x):
    """bf16 bit patterns (uint16) of float32 values, round-to-nearest-even."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    load().oracle_round_bf16(a.reshape(-1), out.reshape(-1), a.size)
    return out


def bf16_to_float(bits):
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(a.shape, dtype=np.float32)
    load().oracle_bf16_to_float(a.reshape(-1), out.reshape(-1), a.size)
    return out

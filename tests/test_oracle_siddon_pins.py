"""Pins of the oracle's cell-constant (Siddon) projector (CPU).

The model (diffct page, Features: matched project/backproject pair for the
cell-constant Siddon model): voxel (i, j, k) is the cube of side one voxel
centred on (i, j, k) in IJK, with constant value; a ray's image is the exact
line integral of that piecewise-constant function.  Pinned by routes that
share nothing with the oracle's plane-crossing merge:

* an explicit system matrix on a small volume, each entry the chord of the
  ray through one voxel's cube from the test-side face-intersection routine
  (tests/pin_math.py): the forward is A x and the backprojection A^T y,
  entry by entry;
* a constant volume: mu times the chord through the cells' box;
* the dot-product identity at a larger size;
* the Beer-Lambert image and its gradient against finite differences.
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests import pin_math as pm

RAW, BL = wl.MODE_RAW, wl.MODE_BEER_LAMBERT


def _exact(w):
    Rt = np.array(w.Rt, dtype=np.float64, copy=True).reshape(-1, 3, 4)
    for b in range(Rt.shape[0]):
        U, _, Vt = np.linalg.svd(Rt[b, :, :3])
        Rt[b, :, :3] = U @ Vt
    w.Rt = Rt
    return w


def _matrix(w):
    """A[ray, voxel] = chord (mm) of the ray through the voxel's cube."""
    nx, ny, nz = w.dims
    sp = np.asarray(w.spacing, np.float64)
    org = np.asarray(w.origin, np.float64)
    A = np.zeros((w.B * w.H * w.W, nx * ny * nz))
    for b in range(w.B):
        for r in range(w.H):
            for c in range(w.W):
                C, d = pm.world_ray(w.K, w.Rt[b].reshape(-1), c, r)
                row = (b * w.H + r) * w.W + c
                for k in range(nz):
                    for j in range(ny):
                        for i in range(nx):
                            centre = org + sp * np.array([i, j, k])
                            ch = pm.box_chord(C, d, centre - 0.5 * sp, centre + 0.5 * sp)
                            if ch is not None:
                                A[row, (k * ny + j) * nx + i] = ch[1] - ch[0]
    return A


def test_siddon_forward_and_backprojection_equal_the_explicit_matrix():
    w = _exact(wl.small_random_case(71, dims=(5, 4, 6), B=2, H=7, W=8))
    df = 0.9
    A = _matrix(w)
    assert np.count_nonzero(A.any(axis=1)) > 40          # most rays hit
    img = oracle.render_siddon(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, df, RAW)
    x = w.vol.reshape(-1).astype(np.float64)
    assert np.allclose(img.reshape(-1), df * (A @ x), rtol=1e-12, atol=1e-12)
    y = np.random.default_rng(3).standard_normal((w.B, w.H, w.W))
    g = oracle.siddon_adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, df, RAW, y)
    assert np.allclose(g.reshape(-1), df * (A.T @ y.reshape(-1)), rtol=1e-12, atol=1e-12)


def test_siddon_constant_volume_gives_mu_times_the_cells_chord():
    w = _exact(wl.small_random_case(72, B=2, H=13, W=11))
    mu = float(np.float32(0.021))
    vol = np.full_like(w.vol, mu)
    img = oracle.render_siddon(vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, 1.0, RAW)
    sp = np.asarray(w.spacing, np.float64)
    lo = np.asarray(w.origin, np.float64) - 0.5 * sp
    hi = lo + np.asarray(w.dims) * sp
    for b in range(w.B):
        for r in range(w.H):
            for c in range(w.W):
                C, d = pm.world_ray(w.K, w.Rt[b].reshape(-1), c, r)
                ch = pm.box_chord(C, d, lo, hi)
                expect = 0.0 if ch is None else mu * (ch[1] - ch[0])
                assert abs(img[b, r, c] - expect) <= 1e-12 + 1e-11 * expect


def test_siddon_dot_product_identity():
    w = wl.small_random_case(73)
    rng = np.random.default_rng(4)
    x = rng.uniform(0, 1, w.vol.shape).astype(np.float32)
    y = rng.standard_normal((w.B, w.H, w.W))
    Ax = oracle.render_siddon(x, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, 1.3, RAW)
    ATy = oracle.siddon_adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, 1.3, RAW, y)
    lhs, rhs = np.sum(Ax * y), np.sum(x.astype(np.float64) * ATy)
    assert abs(lhs - rhs) <= 1e-12 * np.linalg.norm(Ax) * np.linalg.norm(y)


def test_siddon_beer_lambert_and_its_gradient():
    w = wl.small_random_case(74, dims=(8, 7, 9), B=1, H=6, W=7)
    df = 5.0
    raw = oracle.render_siddon(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, df, RAW)
    bl = oracle.render_siddon(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, df, BL)
    assert np.allclose(bl, -np.expm1(-raw), rtol=1e-14, atol=0)
    go = np.random.default_rng(5).standard_normal((1, w.H, w.W))
    g = oracle.siddon_adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, df, BL, go,
                              vol=w.vol)
    delta = np.random.default_rng(6).standard_normal(w.vol.shape)
    h = 1e-4
    vp = (w.vol + h * delta).astype(np.float32)
    vm = (w.vol - h * delta).astype(np.float32)
    fd = np.sum(go * (oracle.render_siddon(vp, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W,
                                           df, BL) -
                      oracle.render_siddon(vm, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W,
                                           df, BL)))
    dv = vp.astype(np.float64) - vm.astype(np.float64)
    assert abs(fd - np.sum(g * dv)) <= 1e-7 * np.sum(np.abs(g * dv))

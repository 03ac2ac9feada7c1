"""Pins of the fp64 oracle against things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle -- a dropped
term, a wrong sign or index, a transposed operand, t in voxels instead of
mm, f and 1-f swapped, a half-pixel shift -- fails at least one of them:

* closed forms: constant volume (chord x mu), linear volume (chord x value
  at the chord midpoint), axis ray through voxel centres (trapezoid rule),
  Beer-Lambert of a known integral;
* brute force: the exact integral of the trilinear interpolant on 8^3,
  with O(N^-2) convergence of the midpoint sum towards it;
* the projection equation x ~ K [R | t] X for the oracle's rays;
* an explicit 8^3 system matrix for the adjoint, the dot-product identity,
  and finite differences for the Beer-Lambert adjoint;
* a voxelised sphere against its analytic chords (units, magnification);
* invariances: mirror, 90-degree rotation, translation, linearity;
* bf16 rounding against torch's CPU conversion.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests import pin_math as pm

RAW, BL = wl.MODE_RAW, wl.MODE_BEER_LAMBERT
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _box_world(w):
    lo = np.asarray(w.origin, dtype=np.float64)
    hi = lo + (np.asarray(w.dims) - 1) * np.asarray(w.spacing, dtype=np.float64)
    return lo, hi


def _render(w, vol=None, mode=None, df=None, Rt=None, K=None, H=None, W=None, N=None):
    return oracle.render(w.vol if vol is None else vol, w.dims, w.spacing, w.origin,
                         w.K if K is None else K, w.Rt if Rt is None else Rt,
                         w.H if H is None else H, w.W if W is None else W,
                         w.n_samples if N is None else N,
                         w.density_factor if df is None else df,
                         w.mode if mode is None else mode)


def _orthonormal(Rt):
    """fp64 copy of [R|t] with each R replaced by its nearest rotation (polar
    factor), so that R^T = R^-1 to fp64 rounding.  The oracle widens whatever
    geometry it is given; the pins want the HZ identities to hold exactly."""
    Rt = np.array(Rt, dtype=np.float64, copy=True).reshape(-1, 3, 4)
    for b in range(Rt.shape[0]):
        U, _, Vt = np.linalg.svd(Rt[b, :, :3])
        Rt[b, :, :3] = U @ Vt
    return Rt


def _exact(w):
    w.Rt = _orthonormal(w.Rt)
    return w


def _axis_camera(axis_row, C):
    """[R|t] whose camera z axis is world ``axis_row`` (a signed unit vector)
    and whose centre is C (exact permutation matrices)."""
    z = np.asarray(axis_row, dtype=np.float64)
    # pick x, y as the remaining axes, keeping det(R) = +1
    a = int(np.argmax(np.abs(z)))
    e = np.eye(3)
    x = e[(a + 1) % 3]
    y = np.cross(z, x)
    R = np.stack([x, y, z])
    assert abs(np.linalg.det(R) - 1.0) < 1e-12
    t = -R @ np.asarray(C, dtype=np.float64)
    return np.concatenate([R, t[:, None]], axis=1)[None].astype(np.float32)


# ---------------------------------------------------------------------------
# ray geometry
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [1, 2, 3])
def test_rays_satisfy_projection_equation(seed):
    # fp64 rotations (the oracle widens whatever it is given), so R^T = R^-1 to 1e-16
    w = wl.small_random_case(seed)
    rng = np.random.default_rng(seed)
    for b in range(w.B):
        Rt = np.empty((3, 4))
        Rt[:, :3] = wl.random_rotation(rng)
        Rt[:, 3] = rng.uniform(-30, 30, size=3) + [0, 0, 150]
        for _ in range(20):
            u, v = rng.uniform(-5, w.W + 5), rng.uniform(-5, w.H + 5)
            hit, Cijk, dijk, t0, t1 = oracle.ray(w.dims, w.spacing, w.origin, w.K, Rt, u, v)
            sp = np.asarray(w.spacing, np.float64)
            # unit direction in world mm
            assert abs(np.linalg.norm(dijk * sp) - 1.0) < 1e-12
            # camera centre solves R C + t = 0
            C = np.asarray(w.origin, np.float64) + sp * Cijk
            assert np.allclose(Rt[:, :3] @ C + Rt[:, 3], 0.0, atol=1e-11)
            for t in (1.0, 100.0, 1000.0):
                X = C + t * dijk * sp
                pu, pv, depth = pm.project(w.K, Rt, X)
                assert depth > 0, "ray must point into the scene (camera +z)"
                assert abs(pu - u) < 1e-8 and abs(pv - v) < 1e-8


def test_pixel_centre_convention_and_principal_point():
    # the principal-point pixel of a centred detector looks straight along camera +z
    K = wl.intrinsics(100.0, 100.0, 3.5, 2.5)
    Rt = _axis_camera([0, 0, 1], [0, 0, -50])[0]
    _, _, d, _, _ = oracle.ray((4, 4, 4), (1, 1, 1), (0, 0, 0), K, Rt, 3.5, 2.5)
    assert np.allclose(d, [0, 0, 1], atol=0)
    # column index is u (x), row index is v (y, growing downwards in camera y)
    _, _, d, _, _ = oracle.ray((4, 4, 4), (1, 1, 1), (0, 0, 0), K, Rt, 4.5, 2.5)
    assert d[0] > 0 and abs(d[1]) < 1e-15
    _, _, d, _, _ = oracle.ray((4, 4, 4), (1, 1, 1), (0, 0, 0), K, Rt, 3.5, 3.5)
    assert d[1] > 0 and abs(d[0]) < 1e-15


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [11, 12, 13])
def test_constant_volume_gives_mu_times_chord(seed):
    w = _exact(wl.small_random_case(seed, H=19, W=23, n_samples=7))
    mu = float(np.float32(0.037))        # the value the volume actually stores
    vol = np.full_like(w.vol, mu)
    img = _render(w, vol=vol, mode=RAW)
    lo, hi = _box_world(w)
    diag = float(np.linalg.norm(hi - lo))
    n_hit = 0
    for b in range(w.B):
        for r in range(w.H):
            for c in range(w.W):
                C, d = pm.world_ray(w.K, w.Rt[b], c, r)
                ch = pm.box_chord(C, d, lo, hi)
                expect = 0.0 if ch is None else w.density_factor * mu * (ch[1] - ch[0])
                n_hit += ch is not None
                assert abs(img[b, r, c] - expect) <= 1e-10 * w.density_factor * mu * diag, (b, r, c)
    assert n_hit > 0.3 * img.size


def test_camera_inside_volume_starts_at_zero():
    dims, sp = (9, 8, 7), np.array([1.0, 1.5, 2.0], np.float32)
    origin = wl.centred_origin(dims, sp)
    Rt = _axis_camera([0, 0, 1], [0.25, 0.5, 0.0])       # camera in the middle of the box
    K = wl.intrinsics(10.0, 10.0, 0.0, 0.0)
    vol = np.full((7, 8, 9), 0.5, np.float32)
    img = oracle.render(vol, dims, sp, origin, K, Rt, 1, 1, 5, 1.0, RAW)
    # the principal ray runs from z = 0 to the far face z = +6 mm
    assert abs(img[0, 0, 0] - 0.5 * 6.0) < 1e-12
    hit, _, _, t0, t1 = oracle.ray(dims, sp, origin, K, Rt[0], 0.0, 0.0)
    assert hit and t0 == 0.0 and abs(t1 - 6.0) < 1e-12


def test_misses_give_zero():
    dims, sp = (8, 8, 8), np.ones(3, np.float32)
    origin = wl.centred_origin(dims, sp)
    vol = np.ones((8, 8, 8), np.float32)
    K = wl.intrinsics(50.0, 50.0, 3.5, 3.5)
    # camera 100 mm in front of the box, looking away from it
    away = _axis_camera([0, 0, -1], [0, 0, -100])
    assert np.all(_render_args(vol, dims, sp, origin, K, away, 8, 8) == 0.0)
    # parallel principal rays beside the box: along +x at y = 10 mm (box is |y| <= 3.5)
    beside = _axis_camera([1, 0, 0], [-100, 10.0, 0])
    out = _render_args(vol, dims, sp, origin, K, beside, 1, 1, cx=0.0, cy=0.0)
    assert out[0, 0, 0] == 0.0
    # a ray along an edge (zero y, z components, on two face planes) is inside
    edge = _axis_camera([1, 0, 0], [-100, 3.5, 3.5])
    hit = oracle.ray(dims, sp, origin, wl.intrinsics(1, 1, 0, 0), edge[0], 0.0, 0.0)[0]
    assert hit
    # a ray touching the box at one corner only (line y = x - 7 in the face z = 3.5):
    # t_near == t_far, a zero-length chord, so a miss
    corner = _axis_camera([1, 0, 0], [-6.5, -13.5, 3.5])
    hit, _, d, t0, t1 = oracle.ray(dims, sp, origin, wl.intrinsics(1, 1, 0, 0), corner[0], 1.0, 0.0)
    assert d[2] == 0.0 and d[0] == d[1] and not hit and t0 == t1


def _render_args(vol, dims, sp, origin, K, Rt, H, W, cx=None, cy=None, N=8):
    if cx is not None:
        K = wl.intrinsics(float(K[0, 0]), float(K[1, 1]), cx, cy)
    return oracle.render(vol, dims, sp, origin, K, Rt, H, W, N, 1.0, RAW)


@pytest.mark.parametrize("axis", [[1, 0, 0], [0, -1, 0], [0, 0, 1]])
@pytest.mark.parametrize("m", [1, 2, 3])
def test_axis_ray_through_voxel_centres_is_trapezoid_rule(axis, m):
    rng = np.random.default_rng(7)
    dims = (11, 9, 13)
    sp = np.array([0.5, 1.0, 2.0], np.float32)
    origin = wl.centred_origin(dims, sp)
    vol = rng.uniform(0, 1, size=(13, 9, 11)).astype(np.float32)
    a = int(np.argmax(np.abs(axis)))
    # pick a voxel-centre line (integer indices on the two other axes)
    idx = [4, 3, 5]
    C = np.asarray(origin, np.float64) + np.asarray(sp, np.float64) * np.array(idx, np.float64)
    C[a] = -500.0 * np.sign(axis[a])
    Rt = _axis_camera(axis, C)
    n = dims[a]
    N = m * (n - 1)
    out = oracle.render(vol, dims, sp, origin, wl.intrinsics(10, 10, 0, 0), Rt, 1, 1, N, 1.0, RAW)
    line = {0: vol[idx[2], idx[1], :], 1: vol[idx[2], :, idx[0]], 2: vol[:, idx[1], idx[0]]}[a]
    line = line.astype(np.float64)
    trap = float(sp[a]) * float(np.sum(0.5 * (line[:-1] + line[1:])))
    assert abs(out[0, 0, 0] - trap) <= 1e-13 * abs(trap)


def test_ray_along_a_face_counts_as_inside():
    # zero direction components with the camera on the slab planes j = 0 and k = 0:
    # only the edge row contributes (the j+1, k+1 corners have weight 0)
    rng = np.random.default_rng(3)
    dims, sp = (7, 5, 6), np.ones(3, np.float32)
    origin = np.zeros(3, np.float32)
    vol = rng.uniform(0, 1, size=(6, 5, 7)).astype(np.float32)
    Rt = _axis_camera([1, 0, 0], [-20.0, 0.0, 0.0])
    N = 2 * (dims[0] - 1)
    out = oracle.render(vol, dims, sp, origin, wl.intrinsics(10, 10, 0, 0), Rt, 1, 1, N, 1.0, RAW)
    line = vol[0, 0, :].astype(np.float64)
    assert abs(out[0, 0, 0] - np.sum(0.5 * (line[:-1] + line[1:]))) < 1e-13


@pytest.mark.parametrize("seed", [21, 22])
def test_linear_volume_gives_chord_times_midpoint_value(seed):
    # trilinear interpolation reproduces affine functions exactly, and the
    # midpoint rule integrates them exactly: I = df * chord * v(chord midpoint)
    w = _exact(wl.small_random_case(seed, H=13, W=17, n_samples=5))
    nx, ny, nz = w.dims
    a0, ax, ay, az = 0.3, 0.011, -0.007, 0.019
    k, j, i = np.meshgrid(np.arange(nz), np.arange(ny), np.arange(nx), indexing="ij")
    vol = (a0 + ax * i + ay * j + az * k).astype(np.float64)
    vol32 = vol.astype(np.float32)     # float32 storage: affine up to 2^-24 relative
    img = _render(w, vol=vol32, mode=RAW)
    lo, hi = _box_world(w)
    sp = np.asarray(w.spacing, np.float64)
    for b in range(w.B):
        for r in range(w.H):
            for c in range(w.W):
                C, d = pm.world_ray(w.K, w.Rt[b], c, r)
                ch = pm.box_chord(C, d, lo, hi)
                if ch is None:
                    assert img[b, r, c] == 0.0 or abs(img[b, r, c]) < 1e-9
                    continue
                pmid = (C + 0.5 * (ch[0] + ch[1]) * d - lo) / sp
                vmid = a0 + ax * pmid[0] + ay * pmid[1] + az * pmid[2]
                expect = w.density_factor * (ch[1] - ch[0]) * vmid
                # float32 storage of the affine values perturbs them by <= 2^-24 relative
                assert abs(img[b, r, c] - expect) <= 1e-6 * abs(expect) + 1e-9, (b, r, c)


def test_beer_lambert_of_known_integral():
    # a ray whose raw integral is ln 2 must give exactly 1/2 in Beer-Lambert mode
    dims, sp = (5, 4, 4), np.ones(3, np.float32)
    origin = np.zeros(3, np.float32)
    vol = np.ones((4, 4, 5), np.float32)
    Rt = _axis_camera([1, 0, 0], [-10.0, 1.0, 2.0])
    df = math.log(2.0) / 4.0                   # chord is 4 mm through a unit volume
    out = oracle.render(vol, dims, sp, origin, wl.intrinsics(1, 1, 0, 0), Rt, 1, 1, 8, df, BL)
    assert abs(out[0, 0, 0] - 0.5) < 1e-15
    raw = oracle.render(vol, dims, sp, origin, wl.intrinsics(1, 1, 0, 0), Rt, 1, 1, 8, df, RAW)
    assert abs(raw[0, 0, 0] - math.log(2.0)) < 1e-15


def test_golden_hand_derived_cases():
    with open(os.path.join(GOLDEN, "hand_derived.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        nx, ny, nz = case["dims"]
        cf = case["volume_coefficients"]          # v = c0 + c1 i + c2 j + c3 k
        k, j, i = np.meshgrid(np.arange(nz), np.arange(ny), np.arange(nx), indexing="ij")
        vol = (cf[0] + cf[1] * i + cf[2] * j + cf[3] * k).astype(np.float32)
        K = np.asarray(case["K"], np.float64)
        Rt = np.asarray(case["Rt"], np.float64)[None]
        r, c = case["pixel"]
        for mode_name, expect in case["expected"].items():
            mode = RAW if mode_name == "raw" else BL
            out = oracle.render(vol, case["dims"], case["spacing"], case["origin"], K, Rt,
                                case["H"], case["W"], case["n_samples"],
                                case["density_factor"], mode)
            assert abs(out[0, r, c] - expect) <= 1e-13 * max(1.0, abs(expect)), (case["name"],
                                                                                mode_name)


# ---------------------------------------------------------------------------
# brute force on 8^3
# ---------------------------------------------------------------------------

def _tiny_case(seed):
    rng = np.random.default_rng(seed)
    dims = (8, 8, 8)
    sp = np.array([1.0, 1.25, 0.75], np.float32)
    origin = wl.centred_origin(dims, sp)
    vol = rng.uniform(0, 1, size=(8, 8, 8)).astype(np.float32)
    R = wl.random_rotation(rng)
    Rt = np.concatenate([R, np.array([[0.3], [-0.2], [40.0]])], axis=1)[None]
    K = wl.intrinsics(60.0, 60.0, 2.0, 2.0)
    return vol, dims, sp, origin, K, Rt


@pytest.mark.parametrize("seed", [31, 32])
def test_midpoint_sum_converges_to_exact_integral(seed):
    vol, dims, sp, origin, K, Rt = _tiny_case(seed)
    u, v = 2.3, 1.7
    C, d = pm.world_ray(K, Rt[0], u, v)
    lo = np.asarray(origin, np.float64)
    hi = lo + (np.asarray(dims) - 1) * np.asarray(sp, np.float64)
    ch = pm.box_chord(C, d, lo, hi)
    assert ch is not None
    P0 = (C - lo) / np.asarray(sp, np.float64)
    D = d / np.asarray(sp, np.float64)
    exact = pm.exact_line_integral(vol, P0, D, ch[0], ch[1])
    Ns = [2 ** e for e in range(5, 12)]
    # render the wanted pixel through a shifted principal point (pixel (0,0) <-> (u, v))
    Ks = wl.intrinsics(60.0, 60.0, 2.0 - u, 2.0 - v)
    errs = []
    for N in Ns:
        out = oracle.render(vol, dims, sp, origin, Ks, Rt, 1, 1, N, 1.0, RAW)[0, 0, 0]
        errs.append(abs(out - exact))
    slope = np.polyfit(np.log(Ns), np.log(np.maximum(errs, 1e-300)), 1)[0]
    assert -2.6 < slope < -1.6, (slope, errs)
    dense = oracle.render(vol, dims, sp, origin, Ks, Rt, 1, 1, 2 ** 16, 1.0, RAW)[0, 0, 0]
    assert abs(dense - exact) <= 1e-8 * abs(exact)


# ---------------------------------------------------------------------------
# adjoint
# ---------------------------------------------------------------------------

def _tiny_system(seed, H=5, W=6, N=16):
    vol, dims, sp, origin, K, Rt = _tiny_case(seed)
    K = wl.intrinsics(25.0, 25.0, (W - 1) / 2, (H - 1) / 2)
    Rt = np.concatenate([Rt, Rt], axis=0)
    rng = np.random.default_rng(seed + 100)
    R2 = wl.random_rotation(rng)
    Rt[1, :, :3] = R2
    return vol, dims, sp, origin, K, Rt, H, W, N


def test_adjoint_is_transpose_of_explicit_matrix():
    vol, dims, sp, origin, K, Rt, H, W, N = _tiny_system(41)
    nvox = int(np.prod(dims))
    df = 0.8
    A = np.zeros((Rt.shape[0] * H * W, nvox))
    e = np.zeros(nvox, np.float32)
    for jv in range(nvox):
        e[:] = 0
        e[jv] = 1
        A[:, jv] = oracle.render(e.reshape(8, 8, 8), dims, sp, origin, K, Rt, H, W, N, df,
                                 RAW).reshape(-1)
    assert np.count_nonzero(A) > 100
    rng = np.random.default_rng(5)
    x = rng.uniform(0, 1, size=nvox).astype(np.float32)
    y = rng.standard_normal(size=A.shape[0])
    Ax = oracle.render(x.reshape(8, 8, 8), dims, sp, origin, K, Rt, H, W, N, df, RAW).reshape(-1)
    assert np.allclose(Ax, A @ x.astype(np.float64), rtol=0, atol=1e-12)
    ATy = oracle.adjoint(dims, sp, origin, K, Rt, H, W, N, df, RAW, y.reshape(-1, H, W))
    assert np.allclose(ATy.reshape(-1), A.T @ y, rtol=0, atol=1e-12)
    lhs, rhs = float(np.dot(Ax, y)), float(np.dot(x.astype(np.float64), ATy.reshape(-1)))
    assert abs(lhs - rhs) <= 1e-12 * np.linalg.norm(Ax) * np.linalg.norm(y)


def test_beer_lambert_adjoint_matches_finite_differences():
    vol, dims, sp, origin, K, Rt, H, W, N = _tiny_system(43, H=4, W=4, N=12)
    vol = (0.2 * vol).astype(np.float32)
    df = 1.3
    rng = np.random.default_rng(9)
    go = rng.standard_normal(size=(Rt.shape[0], H, W))
    g = oracle.adjoint(dims, sp, origin, K, Rt, H, W, N, df, BL, go, vol=vol)

    def loss(v):
        return float(np.sum(go * oracle.render(v, dims, sp, origin, K, Rt, H, W, N, df, BL)))

    picks = np.argsort(-np.abs(g.reshape(-1)))[:6]
    for jv in picks:
        h = 1e-3
        vp = vol.astype(np.float64).reshape(-1).copy()
        vm = vp.copy()
        vp[jv] += h
        vm[jv] -= h
        # the forward is exact in the volume values, so use float64 via a float32-exact step
        fd = (loss(vp.astype(np.float32).reshape(vol.shape)) -
              loss(vm.astype(np.float32).reshape(vol.shape)))
        hh = float(vp.astype(np.float32)[jv]) - float(vm.astype(np.float32)[jv])
        fd /= hh
        assert abs(fd - g.reshape(-1)[jv]) <= 1e-5 * max(1.0, abs(fd)), (jv, fd, g.reshape(-1)[jv])


# ---------------------------------------------------------------------------
# physical units: a voxelised sphere
# ---------------------------------------------------------------------------

def test_sphere_image_matches_analytic_chords():
    dims = (96, 80, 72)
    sp = np.array([1.0, 1.25, 1.5], np.float32)
    origin = wl.centred_origin(dims, sp)
    centre = np.array([4.0, -3.0, 5.0])
    radius, mu = 38.0, 0.02
    sphere = wl.Ellipsoid(centre, np.full(3, radius), np.eye(3), mu)
    vol = wl.voxelize(dims, sp, np.asarray(origin, np.float64), [sphere]).astype(np.float32)
    Rt = np.empty((1, 3, 4))
    Rt[0] = wl.carm_camera(25.0, -10.0, 300.0)
    H = W = 31
    K = wl.intrinsics(80.0, 80.0, 15.0, 15.0)       # the whole disc (radius ~10 px) in frame
    img = oracle.render(vol, dims, sp, origin, K, Rt, H, W, 400, 1.0, RAW)
    worst = 0.0
    for r in range(H):
        for c in range(W):
            C, d = pm.world_ray(K, Rt[0], c, r)
            # analytic chord of the sphere: |C + t d - centre| = radius
            oc = C - centre
            bq = np.dot(oc, d)
            disc = bq * bq - (np.dot(oc, oc) - radius ** 2)
            chord = 2.0 * math.sqrt(disc) if disc > 0 else 0.0
            if chord > radius:                  # away from the blurred rim
                worst = max(worst, abs(img[0, r, c] - mu * chord))
    assert worst > 0.0
    assert worst <= mu * 2.0 * float(np.max(sp)), worst
    # the disc is centred where the sphere centre projects (a half-pixel
    # convention slip would move it by 0.5 px)
    pu, pv, _ = pm.project(K, Rt[0], centre)
    rows, cols = np.mgrid[0:H, 0:W]
    wgt = img[0] ** 4
    assert abs(np.sum(wgt * cols) / np.sum(wgt) - pu) < 0.2
    assert abs(np.sum(wgt * rows) / np.sum(wgt) - pv) < 0.2


# ---------------------------------------------------------------------------
# invariances
# ---------------------------------------------------------------------------

def _sym_case(seed, H=9, W=11):
    rng = np.random.default_rng(seed)
    dims = (10, 12, 8)
    sp = np.array([1.0, 0.8, 1.2], np.float32)
    origin = wl.centred_origin(dims, sp)
    vol = rng.uniform(0, 1, size=(8, 12, 10)).astype(np.float32)
    Rt = np.empty((2, 3, 4))
    Rt[0] = wl.carm_camera(30.0, 10.0, 60.0)
    Rt[1] = wl.carm_camera(-70.0, -25.0, 45.0)
    K = wl.intrinsics(40.0, 40.0, (W - 1) / 2, (H - 1) / 2)
    return vol, dims, sp, origin, K, Rt, H, W


def test_mirror_invariance():
    vol, dims, sp, origin, K, Rt, H, W = _sym_case(51)
    img = oracle.render(vol, dims, sp, origin, K, Rt, H, W, 32, 1.0, RAW)
    S = np.diag([-1.0, 1.0, 1.0])              # mirror world x (volume axis i)
    Rm = np.empty_like(Rt)
    for b in range(2):
        R, t = Rt[b, :, :3], Rt[b, :, 3]
        C = -R.T @ t
        R2 = S @ R @ S                          # mirror the camera's x too: still a rotation
        Rm[b, :, :3] = R2
        Rm[b, :, 3] = -R2 @ (S @ C)
    img_m = oracle.render(np.ascontiguousarray(vol[:, :, ::-1]), dims, sp, origin, K,
                          Rm, H, W, 32, 1.0, RAW)
    assert np.allclose(img_m, img[:, :, ::-1], rtol=0, atol=1e-5 * np.max(img))


def test_rotation_by_90_degrees_with_permuted_axes():
    vol, dims, sp, origin, K, Rt, H, W = _sym_case(52)
    img = oracle.render(vol, dims, sp, origin, K, Rt, H, W, 32, 1.0, RAW)
    Q = wl.rot_z(math.pi / 2)                   # world (x, y, z) -> (-y, x, z)
    Q = np.round(Q)
    nx, ny, nz = dims
    # new volume: v'(X) = v(Q^T X); new x' = -y, y' = x
    vol2 = np.empty((nz, nx, ny), np.float32)
    for k in range(nz):
        for j2 in range(nx):
            for i2 in range(ny):
                vol2[k, j2, i2] = vol[k, ny - 1 - i2, j2]
    dims2 = (ny, nx, nz)
    sp2 = np.array([sp[1], sp[0], sp[2]], np.float32)
    origin2 = wl.centred_origin(dims2, sp2)
    Rt2 = np.empty_like(Rt)
    for b in range(Rt.shape[0]):
        Rt2[b, :, :3] = Rt[b, :, :3] @ Q.T
        Rt2[b, :, 3] = Rt[b, :, 3]
    img2 = oracle.render(vol2, dims2, sp2, origin2, K, Rt2, H, W, 32, 1.0, RAW)
    assert np.allclose(img2, img, rtol=0, atol=1e-5 * np.max(img))


def test_translation_invariance_and_linearity():
    vol, dims, sp, origin, K, Rt, H, W = _sym_case(53)
    img = oracle.render(vol, dims, sp, origin, K, Rt, H, W, 24, 1.0, RAW)
    delta = np.array([3.0, -2.0, 5.0])
    Rt2 = Rt.copy()
    for b in range(Rt.shape[0]):
        Rt2[b, :, 3] = Rt[b, :, 3] - Rt[b, :, :3] @ delta
    img2 = oracle.render(vol, dims, sp, np.asarray(origin, np.float64) + delta, K, Rt2, H, W, 24,
                         1.0, RAW)
    assert np.allclose(img2, img, rtol=0, atol=1e-9 * np.max(img))
    rng = np.random.default_rng(54)
    v2 = rng.uniform(0, 1, size=vol.shape).astype(np.float32)
    a, b = 0.75, 2.0        # exact in float32, so a*vol + b*v2 is formed exactly in fp64
    comb = (a * vol.astype(np.float64) + b * v2.astype(np.float64))
    comb32 = comb.astype(np.float32)
    lin = oracle.render(comb32, dims, sp, origin, K, Rt, H, W, 24, 1.0, RAW)
    ref = a * img + b * oracle.render(v2, dims, sp, origin, K, Rt, H, W, 24, 1.0, RAW)
    assert np.allclose(lin, ref, rtol=0, atol=1e-6 * np.max(ref))
    img_df = oracle.render(vol, dims, sp, origin, K, Rt, H, W, 24, 3.0, RAW)
    assert np.allclose(img_df, 3.0 * img, rtol=1e-14, atol=0)


# ---------------------------------------------------------------------------
# plumbing of the oracle itself
# ---------------------------------------------------------------------------

def test_render_rays_matches_full_image_and_is_thread_count_independent():
    w = wl.small_random_case(61)
    full1 = _render(w)
    full8 = oracle.render(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                          w.density_factor, w.mode, nthreads=7)
    assert np.array_equal(full1, full8)
    rng = np.random.default_rng(0)
    ids = rng.choice(w.rays, size=200, replace=False)
    sub = oracle.render_rays(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W,
                             w.n_samples, w.density_factor, w.mode, ids)
    assert np.array_equal(sub, full1.reshape(-1)[ids])


def test_trilinear_corner_weights():
    vol = np.arange(8, dtype=np.float32).reshape(2, 2, 2)   # v = i + 2 j + 4 k
    pts = np.array([[0, 0, 0], [1, 1, 1], [0.25, 0.5, 0.75], [1, 0, 0], [1.5, 0, 0],
                    [-0.5, 0, 0], [2.0, 0, 0]])
    got = oracle.trilinear(vol, (2, 2, 2), pts)
    # inside: affine reproduction; outside: zero padding blends towards 0
    assert np.allclose(got[:4], [0, 7, 0.25 + 1.0 + 3.0, 1.0], atol=1e-15)
    assert abs(got[4] - 0.5 * 1.0) < 1e-15     # halfway between v(1,0,0)=1 and padding 0
    assert abs(got[5] - 0.5 * 0.0) < 1e-15     # halfway between padding and v(0,0,0)=0
    assert got[6] == 0.0


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(71)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 0.05,
        rng.uniform(-1e30, 1e30, 2000).astype(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 1e-40, -1e-40, 3.4e38], np.float32),
        # exact ties: 1 + 2^-8 (rounds down to even) and 1 + 3*2^-8 (rounds up to even)
        np.array([1.00390625, 1.01171875, -1.00390625], np.float32),
    ])
    ours = oracle.round_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert oracle.round_bf16(np.array([1.00390625], np.float32))[0] == 0x3F80
    assert oracle.round_bf16(np.array([1.01171875], np.float32))[0] == 0x3F82
    nan = oracle.round_bf16(np.array([np.nan], np.float32))
    assert np.isnan(oracle.bf16_to_float(nan))[0]
    back = oracle.bf16_to_float(ours[:100])
    assert np.array_equal(back, torch.from_numpy(x[:100]).to(torch.bfloat16).float().numpy())

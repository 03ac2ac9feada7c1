"""Pins of the oracle's pose gradient against things other than itself (CPU).

The pose gradient is dL/d[R|t] for L = sum(grad_out * image), the 12 entries
of each view's world-to-camera matrix taken as free variables
(flashdrr.rendering API docs, VolumeRaycaster: rendering is differentiable
with respect to the view matrices).  The oracle reaches it by the chain rule;
these pins reach it by other routes:

* central finite differences of the oracle's own forward (a different code
  path: only the forward is differentiated, numerically), on ragged random
  cases in both modes, with the camera outside the box and inside it (where
  the clip's entry point stays at the camera and has no derivative);
* a constant volume, where the image is df * mu * chord: the derivative of
  the chord computed by finite differences of the test-side face-intersection
  routine (tests/pin_math.py), which shares nothing with the oracle's slab
  clip;
* linearity in grad_out, and zero for a zero upstream gradient.
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests import pin_math as pm

RAW, BL = wl.MODE_RAW, wl.MODE_BEER_LAMBERT


def _case(seed, **kw):
    kw.setdefault("dims", (12, 10, 11))
    kw.setdefault("B", 2)
    kw.setdefault("H", 9)
    kw.setdefault("W", 8)
    kw.setdefault("n_samples", 17)
    return wl.small_random_case(seed, **kw)


def _pose_grad(w, Rt, go, mode):
    return oracle.pose_grad(w.vol, w.dims, w.spacing, w.origin, w.K, Rt, w.H, w.W, w.n_samples,
                            w.density_factor, mode, go)


def _fd_pose_grad(w, Rt, go, mode, h_rot=1e-7, h_t=1e-5):
    """Central differences of sum(go * image) in each of the 12 entries.  The
    steps are small because the midpoint sum is only piecewise smooth: a
    sample crossing a voxel face within the step adds a kink."""
    B = Rt.shape[0]
    out = np.zeros((B, 3, 4))
    for b in range(B):
        for r in range(3):
            for c in range(4):
                h = h_t if c == 3 else h_rot
                Rp, Rm = Rt.copy(), Rt.copy()
                Rp[b, r, c] += h
                Rm[b, r, c] -= h
                ip = oracle.render(w.vol, w.dims, w.spacing, w.origin, w.K, Rp, w.H, w.W,
                                   w.n_samples, w.density_factor, mode)
                im = oracle.render(w.vol, w.dims, w.spacing, w.origin, w.K, Rm, w.H, w.W,
                                   w.n_samples, w.density_factor, mode)
                out[b, r, c] = np.sum(go * (ip - im)) / (2 * h)
    return out


@pytest.mark.parametrize("seed", [11, 12, 13])
@pytest.mark.parametrize("mode", [RAW, BL])
def test_pose_gradient_matches_finite_differences(seed, mode):
    w = _case(seed)
    Rt = w.Rt.astype(np.float64).reshape(-1, 3, 4)
    go = np.random.default_rng(seed).standard_normal((w.B, w.H, w.W))
    g = _pose_grad(w, Rt, go, mode)
    fd = _fd_pose_grad(w, Rt, go, mode)
    for b in range(w.B):
        # rotation and translation entries have different units: compare each
        assert np.max(np.abs(g[b, :, :3] - fd[b, :, :3])) <= 1e-6 * np.max(np.abs(fd[b, :, :3]))
        assert np.max(np.abs(g[b, :, 3] - fd[b, :, 3])) <= 1e-5 * np.max(np.abs(fd[b, :, 3]))


@pytest.mark.parametrize("seed", [14, 15])
def test_alpha_pose_gradient_matches_finite_differences(seed):
    # the composite C = sum T_i a_i mu_i (alpha mode) is smooth in the pose
    # between sample-crossings of voxel faces, like the line integral; a large
    # density_factor keeps the opacities far from the linear regime
    w = _case(seed)
    w.density_factor = 30.0
    Rt = w.Rt.astype(np.float64).reshape(-1, 3, 4)
    go = np.random.default_rng(seed).standard_normal((w.B, w.H, w.W))
    g = _pose_grad(w, Rt, go, wl.MODE_ALPHA)
    fd = _fd_pose_grad(w, Rt, go, wl.MODE_ALPHA)
    for b in range(w.B):
        assert np.max(np.abs(g[b, :, :3] - fd[b, :, :3])) <= 1e-6 * np.max(np.abs(fd[b, :, :3]))
        assert np.max(np.abs(g[b, :, 3] - fd[b, :, 3])) <= 1e-5 * np.max(np.abs(fd[b, :, 3]))
    # and it is not the line integral's gradient
    assert np.max(np.abs(g - _pose_grad(w, Rt, go, RAW))) > 1e-3 * np.max(np.abs(g))


def test_pose_gradient_camera_inside_the_volume():
    # camera at the volume centre: every ray starts at t0 = 0
    w = _case(21, B=1, H=11, W=10)
    Rt = w.Rt.astype(np.float64).reshape(-1, 3, 4)
    centre = np.asarray(w.origin, np.float64) + 0.5 * (np.asarray(w.dims) - 1) * np.asarray(
        w.spacing, np.float64)
    centre += np.array([0.37, -0.21, 0.13])       # off the voxel planes
    Rt[0, :, 3] = -Rt[0, :, :3] @ centre           # C = -R^T t = centre
    hit, _, _, t0, _ = oracle.ray(w.dims, w.spacing, w.origin, w.K, Rt[0].reshape(-1), 4.0, 5.0)
    assert hit and t0 == 0.0
    go = np.random.default_rng(5).standard_normal((1, w.H, w.W))
    for mode in (RAW, BL):
        g = _pose_grad(w, Rt, go, mode)
        fd = _fd_pose_grad(w, Rt, go, mode)
        assert np.max(np.abs(g - fd)) <= 2e-6 * np.max(np.abs(fd))


def _ray_as_written(K, R12, u, v):
    """The method's ray with the 12 entries free: C = -R^T t and direction
    R^T K^-1 (u, v, 1), normalised (numpy solve for K^-1).  Off the rotation
    group R^T is not R^-1, so this -- not a solve with R -- is the function
    whose derivative the pose gradient is."""
    Rt = np.asarray(R12, np.float64).reshape(3, 4)
    R, t = Rt[:, :3], Rt[:, 3]
    d = R.T @ np.linalg.solve(np.asarray(K, np.float64).reshape(3, 3), np.array([u, v, 1.0]))
    return -R.T @ t, d / np.linalg.norm(d)


def test_pose_gradient_of_a_constant_volume_is_the_chord_derivative():
    # image = df * mu * (t1 - t0); d(t1 - t0)/dRt by finite differences of the
    # test-side face-intersection chord on the test-side ray
    w = _case(31, B=1, H=7, W=6, n_samples=5)
    mu = float(np.float32(0.03))
    vol = np.full_like(w.vol, mu)
    Rt = w.Rt.astype(np.float64).reshape(-1, 3, 4)
    go = np.random.default_rng(2).standard_normal((1, w.H, w.W))
    g = oracle.pose_grad(vol, w.dims, w.spacing, w.origin, w.K, Rt, w.H, w.W, w.n_samples,
                         w.density_factor, RAW, go)
    lo = np.asarray(w.origin, np.float64)
    hi = lo + (np.asarray(w.dims) - 1) * np.asarray(w.spacing, np.float64)

    def chord_sum(R12):
        s = 0.0
        for r in range(w.H):
            for c in range(w.W):
                C, d = _ray_as_written(w.K, R12, c, r)
                ch = pm.box_chord(C, d, lo, hi)
                if ch is not None:
                    s += go[0, r, c] * (ch[1] - ch[0])
        return s

    expect = np.zeros((3, 4))
    for r in range(3):
        for c in range(4):
            h = 1e-5 if c == 3 else 1e-7
            Rp, Rm = Rt[0].copy(), Rt[0].copy()
            Rp[r, c] += h
            Rm[r, c] -= h
            expect[r, c] = w.density_factor * mu * (chord_sum(Rp) - chord_sum(Rm)) / (2 * h)
    assert np.max(np.abs(g[0, :, :3] - expect[:, :3])) <= 1e-5 * np.max(np.abs(expect[:, :3]))
    assert np.max(np.abs(g[0, :, 3] - expect[:, 3])) <= 1e-5 * np.max(np.abs(expect[:, 3]))


def test_pose_gradient_is_linear_in_the_upstream_gradient():
    w = _case(41)
    Rt = w.Rt.astype(np.float64).reshape(-1, 3, 4)
    rng = np.random.default_rng(9)
    a = rng.standard_normal((w.B, w.H, w.W))
    b = rng.standard_normal((w.B, w.H, w.W))
    ga, gb = _pose_grad(w, Rt, a, BL), _pose_grad(w, Rt, b, BL)
    gab = _pose_grad(w, Rt, 2.0 * a - 3.0 * b, BL)
    assert np.allclose(gab, 2.0 * ga - 3.0 * gb, rtol=1e-12, atol=1e-12 * np.max(np.abs(gab)))
    assert np.all(_pose_grad(w, Rt, np.zeros_like(a), BL) == 0.0)

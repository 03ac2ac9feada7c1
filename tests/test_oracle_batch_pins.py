"""Pins of the oracle's batch rule (CPU): VolumeRaycaster.forward's volumes
(B, C, D, H, W) and view matrices (N, 4, 4), N = B * views_per_vol, N == 1
broadcast to B, output (N, C, H, W) (flashdrr.rendering API docs).

Each volume-channel is a constant with its own value, so every output image
is that value times density_factor times the box chord (tests/pin_math.py):
an image shows by its value which volume and channel, and by its chords
which pose, it was rendered from -- checked against the rule as the page
states it, written here without the oracle's helper.
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests import pin_math as pm


def _case(n_vols, C, n_views, seed):
    w = wl.small_random_case(seed, dims=(9, 8, 10), B=n_views, H=6, W=7, n_samples=11)
    Rt = np.array(w.Rt, np.float64).reshape(-1, 3, 4)
    for b in range(Rt.shape[0]):
        U, _, Vt = np.linalg.svd(Rt[b, :, :3])
        Rt[b, :, :3] = U @ Vt
    vals = np.array([[0.01 * (1 + v + 10 * ch) for ch in range(C)] for v in range(n_vols)],
                    np.float32)
    nx, ny, nz = w.dims
    vols = np.broadcast_to(vals[:, :, None, None, None], (n_vols, C, nz, ny, nx)).copy()
    return w, Rt, vols, vals


@pytest.mark.parametrize("n_vols,C,n_views", [(2, 3, 4), (3, 1, 1), (1, 2, 3), (2, 2, 2)])
def test_batch_rule_by_constant_volumes(n_vols, C, n_views):
    w, Rt, vols, vals = _case(n_vols, C, n_views, 81 + n_views)
    out = oracle.render_batched(vols, w.dims, w.spacing, w.origin, w.K, Rt, n_views, w.H, w.W,
                                w.n_samples, w.density_factor, wl.MODE_RAW)
    n_out = n_vols if (n_views == 1 and n_vols > 1) else n_views
    assert out.shape == (n_out, C, w.H, w.W)
    lo = np.asarray(w.origin, np.float64)
    hi = lo + (np.asarray(w.dims) - 1) * np.asarray(w.spacing, np.float64)
    for n in range(n_out):
        pose = 0 if n_views == 1 else n
        vol = n if (n_views == 1 and n_vols > 1) else n // (n_views // n_vols)
        for r in range(w.H):
            for c in range(w.W):
                C0, d = pm.world_ray(w.K, Rt[pose].reshape(-1), c, r)
                ch_ = pm.box_chord(C0, d, lo, hi)
                chord = 0.0 if ch_ is None else ch_[1] - ch_[0]
                for ch in range(C):
                    expect = w.density_factor * float(vals[vol, ch]) * chord
                    assert abs(out[n, ch, r, c] - expect) <= 1e-12 + 1e-9 * expect


def test_batch_rule_rejects_a_view_count_that_does_not_divide():
    with pytest.raises(AssertionError):
        oracle.batch_map(2, 1, 3)


def test_batched_adjoint_is_the_transpose_of_the_batched_forward():
    w, Rt, _, _ = _case(2, 2, 4, 91)
    rng = np.random.default_rng(3)
    nx, ny, nz = w.dims
    x = rng.uniform(0, 1, (2, 2, nz, ny, nx)).astype(np.float32)
    y = rng.standard_normal((4, 2, w.H, w.W))
    Ax = oracle.render_batched(x, w.dims, w.spacing, w.origin, w.K, Rt, 4, w.H, w.W, w.n_samples,
                               w.density_factor, wl.MODE_RAW)
    ATy = oracle.adjoint_batched(w.dims, w.spacing, w.origin, w.K, Rt, 2, 4, w.H, w.W,
                                 w.n_samples, w.density_factor, wl.MODE_RAW, y)
    lhs, rhs = np.sum(Ax * y), np.sum(x.astype(np.float64) * ATy)
    assert abs(lhs - rhs) <= 1e-12 * np.linalg.norm(Ax) * np.linalg.norm(y)


@pytest.mark.parametrize("n_vols,C,n_views,mode", [(2, 2, 4, wl.MODE_RAW), (3, 1, 1, wl.MODE_BEER_LAMBERT)])
def test_batched_pose_gradient_matches_finite_differences_of_the_batched_render(n_vols, C, n_views,
                                                                                mode):
    # random volume-channels, so that images of one pose differ; central
    # differences of sum(go * render_batched) in each pose entry.  With one
    # pose broadcast to every volume, all images add into pose 0.
    w, Rt, _, _ = _case(n_vols, C, n_views, 95 + n_views)
    nx, ny, nz = w.dims
    rng = np.random.default_rng(11 + n_views)
    vols = rng.uniform(0.0, 0.05, (n_vols, C, nz, ny, nx)).astype(np.float32)
    n_out = n_vols if (n_views == 1 and n_vols > 1) else n_views
    go = rng.standard_normal((n_out, C, w.H, w.W))
    g = oracle.pose_grad_batched(vols, w.dims, w.spacing, w.origin, w.K, Rt, n_views, w.H, w.W,
                                 w.n_samples, w.density_factor, mode, go)
    assert g.shape == (Rt.shape[0], 3, 4)

    def objective(R):
        return np.sum(go * oracle.render_batched(vols, w.dims, w.spacing, w.origin, w.K, R,
                                                 n_views, w.H, w.W, w.n_samples,
                                                 w.density_factor, mode))

    for p in range(Rt.shape[0]):
        fd = np.zeros((3, 4))
        for r in range(3):
            for c in range(4):
                h = 1e-5 if c == 3 else 1e-7
                Rp, Rm = Rt.copy(), Rt.copy()
                Rp[p, r, c] += h
                Rm[p, r, c] -= h
                fd[r, c] = (objective(Rp) - objective(Rm)) / (2 * h)
        assert np.max(np.abs(g[p, :, :3] - fd[:, :3])) <= 1e-6 * np.max(np.abs(fd[:, :3]))
        assert np.max(np.abs(g[p, :, 3] - fd[:, 3])) <= 1e-5 * np.max(np.abs(fd[:, 3]))


def test_batched_alpha_volume_gradient_matches_finite_differences():
    # the alpha composite is not linear in the volume: its batched gradient
    # (adjoint_batched in alpha mode, each image's gradient into its own
    # volume-channel) against central differences of the batched alpha render
    w, Rt, _, _ = _case(2, 2, 4, 97)
    w.density_factor = 30.0
    nx, ny, nz = w.dims
    rng = np.random.default_rng(21)
    vols = rng.uniform(0.0, 0.05, (2, 2, nz, ny, nx)).astype(np.float32)
    go = rng.standard_normal((4, 2, w.H, w.W))
    g = oracle.adjoint_batched(w.dims, w.spacing, w.origin, w.K, Rt, 2, 4, w.H, w.W, w.n_samples,
                               w.density_factor, wl.MODE_ALPHA, go, vols=vols)
    for _ in range(3):
        delta = rng.standard_normal(vols.shape)
        h = 1e-5
        vp = (vols + h * delta).astype(np.float32)
        vm = (vols - h * delta).astype(np.float32)
        dv = vp.astype(np.float64) - vm.astype(np.float64)
        fd = np.sum(go * (oracle.render_batched(vp, w.dims, w.spacing, w.origin, w.K, Rt, 4, w.H,
                                                w.W, w.n_samples, w.density_factor,
                                                wl.MODE_ALPHA) -
                          oracle.render_batched(vm, w.dims, w.spacing, w.origin, w.K, Rt, 4, w.H,
                                                w.W, w.n_samples, w.density_factor,
                                                wl.MODE_ALPHA)))
        assert abs(fd - np.sum(g * dv)) <= 1e-6 * np.sum(np.abs(g * dv))

"""Pins of the oracle's alpha compositing and Gaussian-Poisson surrogate (CPU).

Alpha compositing (flashdrr.rendering API docs, VolumeRaycaster.__init__,
use_beer_lambert = False: front-to-back over operator) is read as the
emission-absorption sum C = sum_i T_i a_i mu_i, a_i = 1 - exp(-df mu_i dt),
T_{i+1} = T_i (1 - a_i).  Pinned by:

* a constant volume: C = mu (1 - exp(-df mu chord)) for any N, the chord from
  the test-side face-intersection routine;
* one sample: C = mu(mid) (1 - exp(-df mu(mid) chord)), mu(mid) from the
  test-side trilinear interpolation at the chord midpoint;
* the continuum limit on a linear ramp along an axis ray: the integral
  df int (m0 + m1 t)^2 exp(-df (m0 t + m1 t^2 / 2)) dt, by scipy quadrature --
  different for the two directions through the ramp, so it pins
  front-to-back order;
* its volume gradient against central finite differences of the oracle's
  alpha image along random directions.

The surrogate (VolumeRaycaster.apply_poisson) on a Beer-Lambert image
1 - T: hand-worked values inside and at both clamps, its mean and variance
over many draws, and its derivative against finite differences.
"""
import math

import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests import pin_math as pm

ALPHA = wl.MODE_ALPHA


def _render(w, vol=None, mode=ALPHA, df=None, N=None, Rt=None):
    return oracle.render(w.vol if vol is None else vol, w.dims, w.spacing, w.origin, w.K,
                         w.Rt if Rt is None else Rt, w.H, w.W, w.n_samples if N is None else N,
                         w.density_factor if df is None else df, mode)


def _exact(w):
    """fp64 poses with each R replaced by its nearest rotation, so that the
    test-side rays (which invert R) and the oracle's (which transpose it)
    are the same lines."""
    Rt = np.array(w.Rt, dtype=np.float64, copy=True).reshape(-1, 3, 4)
    for b in range(Rt.shape[0]):
        U, _, Vt = np.linalg.svd(Rt[b, :, :3])
        Rt[b, :, :3] = U @ Vt
    w.Rt = Rt
    return w


def _box(w):
    lo = np.asarray(w.origin, np.float64)
    return lo, lo + (np.asarray(w.dims) - 1) * np.asarray(w.spacing, np.float64)


@pytest.mark.parametrize("N", [1, 7, 40])
def test_alpha_constant_volume_closed_form(N):
    w = _exact(wl.small_random_case(51, B=2, H=11, W=13))
    mu = float(np.float32(0.04))
    vol = np.full_like(w.vol, mu)
    df = 3.0
    img = _render(w, vol=vol, df=df, N=N)
    lo, hi = _box(w)
    for b in range(w.B):
        for r in range(w.H):
            for c in range(w.W):
                C, d = pm.world_ray(w.K, w.Rt[b].reshape(-1), c, r)
                ch = pm.box_chord(C, d, lo, hi)
                expect = 0.0 if ch is None else mu * (1.0 - math.exp(-df * mu * (ch[1] - ch[0])))
                assert abs(img[b, r, c] - expect) <= 1e-12 + 1e-9 * expect


def test_alpha_one_sample_closed_form():
    w = _exact(wl.small_random_case(52, B=1, H=9, W=10))
    df = 2.5
    img = _render(w, df=df, N=1)
    lo, hi = _box(w)
    sp, org = np.asarray(w.spacing, np.float64), np.asarray(w.origin, np.float64)
    hits = 0
    for r in range(w.H):
        for c in range(w.W):
            C, d = pm.world_ray(w.K, w.Rt[0].reshape(-1), c, r)
            ch = pm.box_chord(C, d, lo, hi)
            if ch is None:
                assert img[0, r, c] == 0.0
                continue
            hits += 1
            mid = C + 0.5 * (ch[0] + ch[1]) * d
            m = pm.trilinear_zero_padded(w.vol, (mid - org) / sp)
            expect = m * (1.0 - math.exp(-df * m * (ch[1] - ch[0])))
            assert abs(img[0, r, c] - expect) <= 1e-12 + 1e-8 * abs(expect)
    assert hits > 20


def test_alpha_continuum_limit_on_a_ramp_pins_front_to_back_order():
    from scipy.integrate import quad
    # volume linear in i: mu = m0 + m1 * i (trilinear reproduces it exactly);
    # axis rays along +x and -x through voxel-centre rows
    nx, ny, nz = 33, 5, 5
    m0, m1 = 0.01, 0.004
    i = np.arange(nx, dtype=np.float64)
    vol = np.broadcast_to((m0 + m1 * i)[None, None, :], (nz, ny, nx)).astype(np.float32)
    spacing = np.array([1.0, 1.0, 1.0], np.float32)
    origin = np.zeros(3, np.float32)
    K = wl.intrinsics(100.0, 100.0, 0.0, 0.0)
    df, N, L = 2.0, 4096, float(nx - 1)
    vals = vol[0, 0, :].astype(np.float64)     # the float32 voxel values
    a0, a1 = vals[0], (vals[-1] - vals[0]) / L

    def continuum(start, slope):
        f = lambda t: df * (start + slope * t) ** 2 * math.exp(-df * (start * t + slope * t * t / 2))
        return quad(f, 0.0, L, epsabs=1e-14, epsrel=1e-12)[0]

    results = []
    for sign in (+1, -1):
        # camera on the x axis at (sign = +1) x = -20 looking along +x, or x = nx + 19 along -x
        Xc = np.array([-20.0 if sign > 0 else L + 20.0, 2.0, 2.0])
        fwd = np.array([float(sign), 0.0, 0.0])
        Rt = wl.look_at_extrinsics(Xc, Xc + fwd, np.array([0.0, 0.0, 1.0]))
        img = oracle.render(vol, (nx, ny, nz), spacing, origin, K,
                            Rt.reshape(1, 3, 4).astype(np.float64), 1, 1, N, df, ALPHA)
        start, slope = (a0, a1) if sign > 0 else (a0 + a1 * L, -a1)
        expect = continuum(start, slope)
        assert abs(img[0, 0, 0] - expect) <= 2e-4 * expect, (sign, img[0, 0, 0], expect)
        results.append(img[0, 0, 0])
    assert abs(results[0] - results[1]) > 1e-2 * results[0]     # the two orders differ


@pytest.mark.parametrize("seed", [61, 62])
def test_alpha_volume_gradient_matches_finite_differences(seed):
    w = wl.small_random_case(seed, dims=(9, 8, 10), B=2, H=7, W=8, n_samples=23)
    df = 40.0          # opacities of order 0.1-1 per sample: far from the linear regime
    rng = np.random.default_rng(seed)
    go = rng.standard_normal((w.B, w.H, w.W))
    g = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples, df,
                       ALPHA, go, vol=w.vol)
    for _ in range(4):
        delta = rng.standard_normal(w.vol.shape)
        h = 1e-5
        vp = (w.vol + h * delta).astype(np.float32)
        vm = (w.vol - h * delta).astype(np.float32)
        # the float32 volumes actually rendered differ by dv, not exactly 2 h delta
        dv = vp.astype(np.float64) - vm.astype(np.float64)
        lhs = np.sum(go * (_render(w, vol=vp, df=df) - _render(w, vol=vm, df=df)))
        rhs = np.sum(g * dv)
        assert abs(lhs - rhs) <= 1e-6 * np.sum(np.abs(g * dv))


def test_alpha_gradient_is_exact_on_a_single_voxel_direction():
    # one voxel changed: the directional derivative equals that voxel's gradient entry
    w = wl.small_random_case(63, dims=(7, 6, 8), B=1, H=6, W=7, n_samples=15)
    df = 25.0
    go = np.random.default_rng(1).standard_normal((1, w.H, w.W))
    g = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples, df,
                       ALPHA, go, vol=w.vol)
    k, j, i = np.unravel_index(np.argmax(np.abs(g)), g.shape)
    vp = w.vol.astype(np.float64).copy()
    vm = vp.copy()
    h = 1e-5
    vp[k, j, i] += h
    vm[k, j, i] -= h
    fd = np.sum(go * (_render(w, vol=vp.astype(np.float32), df=df) -
                      _render(w, vol=vm.astype(np.float32), df=df)))
    hh = float(np.float32(w.vol[k, j, i] + h)) - float(np.float32(w.vol[k, j, i] - h))
    assert abs(fd / hh - g[k, j, i]) <= 1e-5 * abs(g[k, j, i])


# ---------------------------------------------------------------------------
# Gaussian-Poisson surrogate on a Beer-Lambert image 1 - T

def test_noise_hand_values():
    i0 = 100.0
    image = np.array([0.75, 0.75, 0.75, 1.0, 0.0, 0.19])
    z = np.array([1.0, -10.0, 20.0, 3.0, 0.0, -2.0])
    out = oracle.poisson_noise(image, z, i0)
    # T = 0.25: T + sqrt(T/i0) z = 0.25 + 0.05 z
    expect = np.array([1 - 0.30, 1 - 0.0, 1 - 1.0, 1.0, 0.0, 1 - (0.81 - 0.09 * 2)])
    assert np.allclose(out, expect, rtol=0, atol=1e-15)


def test_noise_mean_and_variance():
    rng = np.random.default_rng(8)
    T, i0, n = 0.4, 5000.0, 400000
    z = rng.standard_normal(n)
    out = oracle.poisson_noise(np.full(n, 1.0 - T), z, i0)
    Tn = 1.0 - out
    assert abs(Tn.mean() - T) <= 5 * math.sqrt(T / i0 / n)
    assert abs(Tn.var() / (T / i0) - 1.0) <= 0.02


def test_noise_derivative_matches_finite_differences():
    rng = np.random.default_rng(9)
    n = 2000
    image = rng.uniform(0.0, 0.98, n)
    z = rng.standard_normal(n) * 2.0
    i0 = 30.0
    go = rng.standard_normal(n)
    g = oracle.poisson_noise_backward(image, z, i0, go)
    h = 1e-7
    fd = (oracle.poisson_noise(image + h, z, i0) - oracle.poisson_noise(image - h, z, i0)) / (2 * h)
    # away from the clamps (where the derivative jumps) they agree
    T = 1.0 - image
    Tn = T + np.sqrt(T / i0) * z
    smooth = (np.abs(Tn) > 1e-4) & (np.abs(Tn - 1.0) > 1e-4)
    assert smooth.sum() > 1500
    assert np.allclose(g[smooth], go[smooth] * fd[smooth], rtol=1e-6, atol=1e-8)
    clamped = (Tn <= 0.0) | (Tn >= 1.0)
    assert clamped.sum() > 10 and np.all(g[clamped] == 0.0)

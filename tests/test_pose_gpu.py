"""GPU parity of the pose gradient dL/d[R|t] (drr_render_pose_grad; line
integral, Beer-Lambert and alpha composite) against
the fp64 oracle's, which tests/test_oracle_pose_pins.py pins to finite
differences and to a constant-volume closed form.

Tolerance.  No page fixes one.  The kernel sums the value, gradient and
index-weighted gradient of the interpolant along each ray in fp32 (like the
forward's sum), forms each ray's 12 terms in fp64 and sums CTAs with fp32
atomics; the per-view entries are sums over many rays whose terms cancel in
part.  Read per view, for the rotation block and the translation column
separately (different units): normwise max|gpu - oracle| / max|oracle|
<= 1e-4 for fp32 volumes, and for bf16 volumes against the oracle fed the
same bf16-rounded values.
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import (BF16, CORNERS, F32, LAYOUTS, LINEAR, PADDED, QUADS,
                               assert_pose_parity, bf16_values, gpu_forward, gpu_pose_grad)

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _oracle(w, go, mode, vol=None, nthreads=8):
    return oracle.pose_grad(w.vol if vol is None else vol, w.dims, w.spacing, w.origin, w.K,
                            w.Rt, w.H, w.W, w.n_samples, w.density_factor, mode, go,
                            nthreads=nthreads)


@pytest.mark.parametrize("seed", [301, 302])
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_pose_gradient_small_ragged(cuda, seed, mode, layout):
    w = wl.small_random_case(seed)
    go = np.random.default_rng(seed).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=layout, dtype=F32, mode=mode) if mode else None
    got = gpu_pose_grad(w, go, layout=layout, dtype=F32, mode=mode, fwd_out=fwd)
    assert_pose_parity(got, _oracle(w, go, mode), TOL, what=f"seed {seed} layout {layout}")


@pytest.mark.parametrize("layout", LAYOUTS)
def test_pose_gradient_bf16_volume(cuda, layout):
    w = wl.small_random_case(303)
    go = np.random.default_rng(3).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    got = gpu_pose_grad(w, go, layout=layout, dtype=BF16, mode=wl.MODE_RAW)
    ref = _oracle(w, go, wl.MODE_RAW, vol=bf16_values(w.vol))
    assert_pose_parity(got, ref, TOL, what=f"bf16 layout {layout}")


@pytest.mark.parametrize("seed", [311, 312])
@pytest.mark.parametrize("layout,dtype", [(LINEAR, F32), (PADDED, F32), (CORNERS, BF16),
                                          (QUADS, F32)])
def test_alpha_pose_gradient_small_ragged(cuda, seed, layout, dtype):
    # the composite's pose gradient: samples weighted by dC/dmu_i, dt through
    # the opacities; opacities far from the linear regime
    w = wl.small_random_case(seed)
    w.density_factor = 30.0
    go = np.random.default_rng(seed).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=layout, dtype=dtype, mode=wl.MODE_ALPHA)
    got = gpu_pose_grad(w, go, layout=layout, dtype=dtype, mode=wl.MODE_ALPHA, fwd_out=fwd)
    vol = bf16_values(w.vol) if dtype == BF16 else None
    ref = _oracle(w, go, wl.MODE_ALPHA, vol=vol)
    assert_pose_parity(got, ref, TOL, what=f"alpha seed {seed} layout {layout} dtype {dtype}")


@pytest.mark.slow
def test_alpha_pose_gradient_config3_sparse_upstream(cuda):
    w = wl.make_config(3)
    w.density_factor = 10.0
    rng = np.random.default_rng(37)
    go = np.zeros((w.B, w.H, w.W), np.float32)
    ids = rng.choice(w.rays, size=2000, replace=False)
    go.reshape(-1)[ids] = rng.standard_normal(2000).astype(np.float32)
    fwd = gpu_forward(w, layout=CORNERS, dtype=BF16, mode=wl.MODE_ALPHA)
    got = gpu_pose_grad(w, go, layout=CORNERS, dtype=BF16, mode=wl.MODE_ALPHA, fwd_out=fwd)
    ref = _oracle(w, go, wl.MODE_ALPHA, vol=bf16_values(w.vol), nthreads=4)
    assert_pose_parity(got, ref, TOL, what="alpha, config 3, 2000 rays")


def test_pose_gradient_camera_inside_the_volume(cuda):
    w = wl.small_random_case(304, B=1)
    Rt = w.Rt.astype(np.float64).reshape(-1, 3, 4)
    centre = np.asarray(w.origin, np.float64) + 0.5 * (np.asarray(w.dims) - 1) * np.asarray(
        w.spacing, np.float64) + np.array([0.37, -0.21, 0.13])
    Rt[0, :, 3] = -Rt[0, :, :3] @ centre
    w.Rt = Rt.astype(np.float32)
    go = np.random.default_rng(4).standard_normal((1, w.H, w.W)).astype(np.float32)
    got = gpu_pose_grad(w, go, layout=PADDED, dtype=F32, mode=wl.MODE_RAW)
    assert_pose_parity(got, _oracle(w, go, wl.MODE_RAW), TOL, what="camera inside")


def test_pose_gradient_accumulates_and_skips_zero_gradient(cuda):
    w = wl.small_random_case(305)
    go = np.random.default_rng(5).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    once = gpu_pose_grad(w, go, mode=wl.MODE_RAW)
    twice = gpu_pose_grad(w, go, mode=wl.MODE_RAW, accumulate=once.astype(np.float32))
    assert np.allclose(twice, 2 * once, rtol=1e-5, atol=1e-6 * np.abs(once).max())
    zero = gpu_pose_grad(w, np.zeros_like(go), mode=wl.MODE_RAW)
    assert np.all(zero == 0.0)


@pytest.mark.slow
def test_pose_gradient_config3_sparse_upstream(cuda):
    # the 1024^2 x 512 C-arm geometry (bf16 corner records, Beer-Lambert) with
    # the oracle on 2000 random rays of upstream gradient
    w = wl.make_config(3)
    rng = np.random.default_rng(36)
    go = np.zeros((w.B, w.H, w.W), np.float32)
    ids = rng.choice(w.rays, size=2000, replace=False)
    go.reshape(-1)[ids] = rng.standard_normal(2000).astype(np.float32)
    fwd = gpu_forward(w, layout=CORNERS, dtype=BF16, mode=w.mode)
    got = gpu_pose_grad(w, go, layout=CORNERS, dtype=BF16, mode=w.mode, fwd_out=fwd)
    ref = _oracle(w, go, w.mode, vol=bf16_values(w.vol), nthreads=4)
    assert_pose_parity(got, ref, TOL, what="config 3, 2000 rays")


@pytest.mark.slow
def test_pose_gradient_config2_full(cuda):
    # 64 views x 200^2 x 256 samples, fp32 corner records, every ray
    w = wl.make_config(2)
    w.Rt = w.Rt[:8]
    go = np.random.default_rng(22).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=CORNERS, dtype=F32, mode=w.mode)
    got = gpu_pose_grad(w, go, layout=CORNERS, dtype=F32, mode=w.mode, fwd_out=fwd)
    assert_pose_parity(got, _oracle(w, go, w.mode, nthreads=8), TOL, what="config 2, 8 views")


# 32 contiguous full detector rows of every view at the 1024^2 x 512 C-arm
# geometry (rows 472-503: two ragged 16-row tiles around a whole one), every
# ray live, so each CTA's reduction sums full tiles.
POSE_BAND_ROWS = slice(472, 504)


@pytest.mark.slow
@pytest.mark.parametrize("mode", [wl.MODE_BEER_LAMBERT, wl.MODE_ALPHA])
def test_pose_gradient_config3_dense_band(cuda, mode):
    w = wl.make_config(3)
    if mode == wl.MODE_ALPHA:
        w.density_factor = 10.0
    go = np.zeros((w.B, w.H, w.W), np.float32)
    n = POSE_BAND_ROWS.stop - POSE_BAND_ROWS.start
    go[:, POSE_BAND_ROWS, :] = np.random.default_rng(38 + mode).standard_normal(
        (w.B, n, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=CORNERS, dtype=BF16, mode=mode)
    got = gpu_pose_grad(w, go, layout=CORNERS, dtype=BF16, mode=mode, fwd_out=fwd)
    ref = _oracle(w, go, mode, vol=bf16_values(w.vol), nthreads=4)
    assert_pose_parity(got, ref, TOL, what=f"config 3 dense band, mode {mode}")

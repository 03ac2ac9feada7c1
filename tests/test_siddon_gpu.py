"""GPU parity of the cell-constant (Siddon) projector and its matched
backprojection (drr_render_siddon / drr_render_siddon_adjoint) against the
pinned fp64 oracle (tests/test_oracle_siddon_pins.py).

Tolerances: the walk keeps its plane parameters in fp64 and sums length x
value in fp32 (one term per cell crossed), so the forward's bar holds:
1e-4 normwise and per pixel (1e-4 against the oracle fed bf16-rounded
values for bf16 volumes).  The backprojection keeps the adjoint's bar
(normwise max and relative L2 1e-4), and the GPU pair passes the
dot-product identity at 1e-5.
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import (BF16, F32, assert_parity, bf16_values, gpu_siddon,
                               gpu_siddon_adjoint)

pytestmark = pytest.mark.gpu
RAW, BL = wl.MODE_RAW, wl.MODE_BEER_LAMBERT


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _ref(w, mode, vol=None):
    return oracle.render_siddon(w.vol if vol is None else vol, w.dims, w.spacing, w.origin, w.K,
                                w.Rt, w.H, w.W, w.density_factor, mode)


@pytest.mark.parametrize("seed", [501, 502, 503])
@pytest.mark.parametrize("mode", [RAW, BL])
def test_siddon_forward_small_ragged(cuda, seed, mode):
    w = wl.small_random_case(seed)
    assert_parity(gpu_siddon(w, mode=mode), _ref(w, mode), 1e-4, what=f"seed {seed} mode {mode}")


def test_siddon_forward_bf16(cuda):
    w = wl.small_random_case(504)
    assert_parity(gpu_siddon(w, dtype=BF16, mode=RAW), _ref(w, RAW, vol=bf16_values(w.vol)), 1e-4,
                  what="bf16")


def test_siddon_camera_inside_and_along_an_axis(cuda):
    # a camera inside the box (rays start at t0 = 0), and a pose whose optical
    # axis runs along a volume axis (rays nearly parallel to two sets of planes)
    w = wl.small_random_case(505, B=2)
    Rt = w.Rt.astype(np.float64).reshape(-1, 3, 4)
    centre = np.asarray(w.origin, np.float64) + 0.5 * (np.asarray(w.dims) - 1) * np.asarray(
        w.spacing, np.float64) + np.array([0.31, -0.27, 0.19])
    Rt[0, :, 3] = -Rt[0, :, :3] @ centre
    Rt[1] = wl.look_at_extrinsics(centre + np.array([0.0, 0.0, -200.0]), centre,
                                  np.array([0.0, 1.0, 0.0]))
    w.Rt = Rt.astype(np.float32)
    for mode in (RAW, BL):
        assert_parity(gpu_siddon(w, mode=mode), _ref(w, mode), 1e-4, what=f"inside/axis {mode}")


@pytest.mark.parametrize("mode", [RAW, BL])
def test_siddon_backprojection_small_ragged(cuda, mode):
    w = wl.small_random_case(511)
    go = np.random.default_rng(11).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_siddon(w, mode=mode) if mode == BL else None
    got = gpu_siddon_adjoint(w, go, mode=mode, fwd_out=fwd).astype(np.float64)
    ref = oracle.siddon_adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W,
                                w.density_factor, mode, go, vol=w.vol)
    scale = np.max(np.abs(ref))
    assert np.max(np.abs(got - ref)) <= 1e-4 * scale
    assert np.linalg.norm(got - ref) <= 1e-4 * np.linalg.norm(ref)


@pytest.mark.parametrize("cfg", [2, 3])
def test_siddon_dot_product_identity(cuda, cfg):
    w = wl.make_config(cfg)
    if cfg == 2:
        w.Rt = w.Rt[:16]
    rng = np.random.default_rng(cfg)
    x = rng.uniform(0, 1, w.vol.shape).astype(np.float32)
    y = rng.standard_normal((w.B, w.H, w.W)).astype(np.float32)
    Ax = gpu_siddon(w, mode=RAW, vol=x).astype(np.float64)
    ATy = gpu_siddon_adjoint(w, y, mode=RAW).astype(np.float64)
    lhs = float(np.dot(Ax.reshape(-1), y.reshape(-1).astype(np.float64)))
    rhs = float(np.dot(x.reshape(-1).astype(np.float64), ATy.reshape(-1)))
    assert abs(lhs - rhs) <= 1e-5 * np.linalg.norm(Ax) * np.linalg.norm(y.astype(np.float64))


@pytest.mark.slow
def test_siddon_config2_views_against_the_oracle(cuda):
    w = wl.make_config(2)
    w.Rt = w.Rt[:4]
    assert_parity(gpu_siddon(w, dtype=F32, mode=w.mode), _ref(w, w.mode), 1e-4, what="config 2")

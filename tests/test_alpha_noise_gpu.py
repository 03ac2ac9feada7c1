"""GPU parity of front-to-back alpha compositing (DRR_MODE_ALPHA: drr_render
and drr_render_alpha_adjoint, with or without a workspace) and of the
Gaussian-Poisson surrogate (drr_poisson_noise and its backward) against the
pinned fp64 oracle (tests/test_oracle_alpha_noise_pins.py).

Tolerances, read from the arithmetic (no page fixes one): the alpha image
composites in fp32 -- a transmittance product and a running sum over N
samples, the forward's own sample values -- so the forward's bar of 1e-4
(normwise and per pixel) holds for it; its volume gradient keeps the
adjoint's bar (normwise max and relative L2 1e-4), against the oracle fed
the same bf16-rounded values for bf16 volumes.  The surrogate is one fp32
square root and fma per pixel on values in [0, 1]: 1e-6 absolute for the
image; its derivative 1e-5 relative, except within 1e-5 of a clamp, where
fp32 and fp64 may decide the clamp differently and only the zero-or-not
choice is compared away from it.
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import drr
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import (BF16, BRICKS, CORNERS, F32, LAYOUTS, LINEAR, QUADS, assert_parity, bf16_values,
                               gpu_alpha_adjoint, gpu_forward)

pytestmark = pytest.mark.gpu
ALPHA = wl.MODE_ALPHA


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _oracle_image(w, vol=None):
    return oracle.render(w.vol if vol is None else vol, w.dims, w.spacing, w.origin, w.K, w.Rt,
                         w.H, w.W, w.n_samples, w.density_factor, ALPHA)


def _assert_adjoint(got, ref, what):
    got = np.asarray(got, np.float64)
    scale = np.max(np.abs(ref))
    norm = np.max(np.abs(got - ref)) / scale
    l2 = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert norm <= 1e-4 and l2 <= 1e-4, f"{what}: normwise {norm:.3g}, L2 {l2:.3g}"


@pytest.mark.parametrize("df", [0.7, 40.0])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_alpha_forward_small_ragged(cuda, layout, df):
    w = wl.small_random_case(401)
    w.density_factor = df
    got = gpu_forward(w, layout=layout, dtype=F32, mode=ALPHA)
    assert_parity(got, _oracle_image(w), 1e-4, what=f"alpha layout {layout} df {df}")


# bf16 volumes take the series / __expf opacity: with df 0.7 every sample's
# s mu is below 1/8 (the series), with df 20 they spread to about 1 (both)
@pytest.mark.parametrize("df", [0.7, 20.0])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_alpha_forward_bf16(cuda, layout, df):
    w = wl.small_random_case(402)
    w.density_factor = df
    got = gpu_forward(w, layout=layout, dtype=BF16, mode=ALPHA)
    assert_parity(got, _oracle_image(w, vol=bf16_values(w.vol)), 1e-4,
                  what=f"bf16 layout {layout} df {df}")


@pytest.mark.slow
def test_alpha_forward_config2_views(cuda):
    w = wl.make_config(2)
    w.Rt = w.Rt[:6]
    w.density_factor = 30.0
    got = gpu_forward(w, layout=CORNERS, dtype=F32, mode=ALPHA)
    assert_parity(got, _oracle_image(w), 1e-4, what="config 2, 6 views")


@pytest.mark.parametrize("seed", [411, 412])
@pytest.mark.parametrize("layout,dtype", [(LINEAR, F32), (CORNERS, F32), (QUADS, F32),
                                          (BRICKS, F32), (LINEAR, BF16), (CORNERS, BF16),
                                          (QUADS, BF16), (BRICKS, BF16)])
def test_alpha_adjoint_small_ragged(cuda, seed, layout, dtype):
    w = wl.small_random_case(seed)
    w.density_factor = 25.0
    go = np.random.default_rng(seed).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=layout, dtype=dtype, mode=ALPHA)
    got = gpu_alpha_adjoint(w, go, fwd, layout=layout, dtype=dtype)
    vol = bf16_values(w.vol) if dtype == BF16 else w.vol
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, ALPHA, go, vol=vol, nthreads=8)
    _assert_adjoint(got, ref, f"seed {seed} layout {layout} dtype {dtype}")


# rays much closer than a voxel (the geometry of the adjoint's record-path
# tests): with a workspace these views take alpha_records_kernel
DENSE = dict(dims=(23, 17, 29), H=150, W=170, n_samples=40)


@pytest.mark.parametrize("layout,dtype", [(LINEAR, F32), (CORNERS, BF16), (QUADS, F32),
                                          (QUADS, BF16), (BRICKS, F32)])
def test_alpha_adjoint_dense_views_take_the_record_path(cuda, layout, dtype):
    w = wl.small_random_case(421, **DENSE)
    w.density_factor = 25.0
    go = np.random.default_rng(421).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=layout, dtype=dtype, mode=ALPHA)
    vol = bf16_values(w.vol) if dtype == BF16 else w.vol
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, ALPHA, go, vol=vol, nthreads=8)
    for workspace in (False, True):
        got = gpu_alpha_adjoint(w, go, fwd, layout=layout, dtype=dtype, workspace=workspace)
        _assert_adjoint(got, ref, f"dense layout {layout} dtype {dtype} workspace {workspace}")


def test_alpha_adjoint_mixed_dense_and_sparse_views(cuda):
    # the dense geometry with its last view moved 4x farther: two views on the
    # record path, one on the direct path, in one call
    w = wl.small_random_case(423, **DENSE)
    Rt = w.Rt.copy()
    Rt[2, :, 3] *= 4.0
    w.Rt = Rt
    w.density_factor = 25.0
    go = np.random.default_rng(423).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=QUADS, dtype=F32, mode=ALPHA)
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, ALPHA, go, vol=w.vol, nthreads=8)
    got = gpu_alpha_adjoint(w, go, fwd, layout=QUADS, dtype=F32, workspace=True)
    _assert_adjoint(got, ref, "mixed dense and sparse views")


def test_alpha_adjoint_workspace_on_sparse_views(cuda):
    # views the plan leaves sparse still go through the direct kernel
    w = wl.small_random_case(422)
    w.density_factor = 25.0
    go = np.random.default_rng(422).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=CORNERS, dtype=F32, mode=ALPHA)
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, ALPHA, go, vol=w.vol, nthreads=8)
    got = gpu_alpha_adjoint(w, go, fwd, layout=CORNERS, dtype=F32, workspace=True)
    _assert_adjoint(got, ref, "sparse views with a workspace")


@pytest.mark.slow
def test_alpha_adjoint_config3_sparse_upstream(cuda):
    w = wl.make_config(3)
    w.density_factor = 10.0
    rng = np.random.default_rng(37)
    go = np.zeros((w.B, w.H, w.W), np.float32)
    ids = rng.choice(w.rays, size=3000, replace=False)
    go.reshape(-1)[ids] = rng.standard_normal(3000).astype(np.float32)
    fwd = gpu_forward(w, layout=CORNERS, dtype=BF16, mode=ALPHA)
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, ALPHA, go, vol=bf16_values(w.vol), nthreads=4)
    for workspace in (False, True):
        got = gpu_alpha_adjoint(w, go, fwd, layout=CORNERS, dtype=BF16, workspace=workspace)
        _assert_adjoint(got, ref, f"config 3, 3000 rays, workspace {workspace}")


@pytest.mark.slow
def test_alpha_adjoint_config3_dense_band(cuda):
    # the alpha gradient with a workspace as the throughput run's widened row
    # times it (bf16 corner records, 4 views of 1024^2 x 512, every view dense:
    # the moment records of alpha_records_kernel), on a band of 96 full
    # detector rows per view with a dense N(0, 1) upstream gradient
    w = wl.make_config(3)
    go = np.zeros((w.B, w.H, w.W), np.float32)
    go[:, 472:568, :] = np.random.default_rng(38).standard_normal((w.B, 96, w.W)).astype(
        np.float32)
    fwd = gpu_forward(w, layout=CORNERS, dtype=BF16, mode=ALPHA)
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, ALPHA, go, vol=bf16_values(w.vol), nthreads=16)
    got = gpu_alpha_adjoint(w, go, fwd, layout=CORNERS, dtype=BF16, workspace=True)
    _assert_adjoint(got, ref, "config 3 dense band, workspace")


def _noise_inputs(n, seed):
    rng = np.random.default_rng(seed)
    image = rng.uniform(0.0, 1.0, n).astype(np.float32)
    image[: n // 50] = 1.0                      # fully absorbed: T = 0
    image[n // 50: n // 25] = 0.0               # unattenuated: T = 1
    z = (rng.standard_normal(n) * 3.0).astype(np.float32)   # wide: many clamped pixels
    return image, z


@pytest.mark.parametrize("n", [1, 1000, 100003])
def test_noise_forward(cuda, n):
    import torch
    image, z = _noise_inputs(n, n)
    i0 = 50.0
    ref = oracle.poisson_noise(image, z, i0)
    di, dz = torch.from_numpy(image).cuda(), torch.from_numpy(z).cuda()
    out = torch.empty_like(di)
    drr.drr_poisson_noise(di, dz, i0, out)
    drr.drr_poisson_noise(di, dz, i0, di)       # in place
    torch.cuda.synchronize()
    assert np.max(np.abs(out.cpu().numpy() - ref)) <= 1e-6
    assert np.array_equal(di.cpu().numpy(), out.cpu().numpy())


def test_noise_backward(cuda):
    import torch
    n = 200003
    image, z = _noise_inputs(n, 7)
    i0 = 50.0
    go = np.random.default_rng(8).standard_normal(n).astype(np.float32)
    ref = oracle.poisson_noise_backward(image, z, i0, go)
    dgo = torch.from_numpy(go).cuda()
    gi = torch.empty_like(dgo)
    drr.drr_poisson_noise_backward(torch.from_numpy(image).cuda(), torch.from_numpy(z).cuda(), i0,
                                   dgo, gi)
    torch.cuda.synchronize()
    got = gi.cpu().numpy().astype(np.float64)
    T = 1.0 - image.astype(np.float64)
    Tn = T + np.sqrt(np.maximum(T, 0.0) / i0) * z
    far = (np.abs(Tn) > 1e-5) & (np.abs(Tn - 1.0) > 1e-5) & (T > 1e-6)
    assert far.sum() > n // 2
    assert np.allclose(got[far], ref[far], rtol=1e-5, atol=1e-6 * np.abs(ref[far]).max())
    clamped = far & ((Tn < 0.0) | (Tn > 1.0))
    assert clamped.sum() > n // 50 and np.all(got[clamped] == 0.0)
    assert np.all(got[T <= 0.0] == 0.0)           # fully absorbed pixels

"""GPU parity of the batched forward, adjoint and pose gradient
(drr_render_batched / drr_render_adjoint_batched, with or without a
workspace / drr_render_pose_grad_batched) against the oracle's batch rule
(tests/test_oracle_batch_pins.py): volumes x channels x views with the
views grouped per volume, and one view broadcast to every volume.  Each
image carries the single-image tolerances (forward 1e-4 normwise and per
pixel; adjoint 1e-4 normwise and L2, per volume-channel), and the batched
pair passes the dot-product identity at 1e-5.
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import drr
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import (BF16, CORNERS, F32, LAYOUTS, LINEAR, PADDED, QUADS, assert_parity,
                               assert_pose_parity, bf16_values)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _batch(n_vols, C, n_views, seed):
    w = wl.small_random_case(seed, B=n_views)
    nx, ny, nz = w.dims
    vols = np.random.default_rng(seed).uniform(0.0, 0.05, (n_vols, C, nz, ny, nx)).astype(np.float32)
    return w, vols


def _gpu_batched(w, vols, n_views, layout, mode):
    import torch
    n_vols, C = vols.shape[:2]
    v32 = torch.from_numpy(vols).cuda()
    per = drr.drr_prepared_bytes(w.dims, F32, layout)
    if layout == LINEAR:
        src = v32
    else:
        src = torch.empty(n_vols * C * per, dtype=torch.uint8, device="cuda")
        for s in range(n_vols * C):
            drr.drr_prepare_volume(v32.view(n_vols * C, -1)[s], w.dims, F32, layout,
                                   src[s * per:(s + 1) * per], per)
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    n_out = n_vols if (n_views == 1 and n_vols > 1) else n_views
    out = torch.full((n_out, C, w.H, w.W), float("nan"), device="cuda")
    drr.drr_render_batched(src, F32, layout, w.dims, w.spacing, w.origin, w.K, Rt, n_vols, C,
                           n_views, w.H, w.W, w.n_samples, w.density_factor, mode, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _gpu_adjoint_batched(w, n_vols, C, n_views, go, mode, fwd=None, workspace=False):
    import torch
    nx, ny, nz = w.dims
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    g = torch.zeros((n_vols, C, nz, ny, nx), device="cuda")
    fo = None if fwd is None else torch.from_numpy(np.ascontiguousarray(fwd, np.float32)).cuda()
    go_d = torch.from_numpy(np.ascontiguousarray(go, np.float32)).cuda()
    if workspace:
        nbytes = drr.drr_adjoint_batched_workspace_bytes(w.dims, n_vols, C, n_views)
        ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")   # garbage on entry
        drr.drr_render_adjoint_batched_ws(w.dims, w.spacing, w.origin, w.K, Rt, n_vols, C, n_views,
                                          w.H, w.W, w.n_samples, w.density_factor, mode, go_d, fo,
                                          g, ws)
    else:
        drr.drr_render_adjoint_batched(w.dims, w.spacing, w.origin, w.K, Rt, n_vols, C, n_views,
                                       w.H, w.W, w.n_samples, w.density_factor, mode, go_d, fo, g)
    torch.cuda.synchronize()
    return g.cpu().numpy()


@pytest.mark.parametrize("n_vols,C,n_views", [(2, 3, 4), (3, 2, 1), (1, 2, 3)])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_batched_forward(cuda, n_vols, C, n_views, layout):
    w, vols = _batch(n_vols, C, n_views, 601 + n_views)
    got = _gpu_batched(w, vols, n_views, layout, wl.MODE_BEER_LAMBERT)
    ref = oracle.render_batched(vols, w.dims, w.spacing, w.origin, w.K, w.Rt, n_views, w.H, w.W,
                                w.n_samples, w.density_factor, wl.MODE_BEER_LAMBERT)
    assert got.shape == ref.shape
    for n in range(ref.shape[0]):
        for ch in range(C):
            assert_parity(got[n, ch], ref[n, ch], 1e-4, what=f"image ({n}, {ch})")


@pytest.mark.parametrize("n_vols,C,n_views", [(2, 3, 4), (3, 2, 1)])
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
def test_batched_adjoint(cuda, n_vols, C, n_views, mode):
    w, vols = _batch(n_vols, C, n_views, 611 + n_views)
    n_out = n_vols if (n_views == 1 and n_vols > 1) else n_views
    go = np.random.default_rng(5).standard_normal((n_out, C, w.H, w.W)).astype(np.float32)
    fwd = _gpu_batched(w, vols, n_views, PADDED, mode) if mode else None
    got = _gpu_adjoint_batched(w, n_vols, C, n_views, go, mode, fwd)
    ref = oracle.adjoint_batched(w.dims, w.spacing, w.origin, w.K, w.Rt, n_vols, n_views, w.H,
                                 w.W, w.n_samples, w.density_factor, mode, go, vols=vols,
                                 nthreads=4)
    for v in range(n_vols):
        for ch in range(C):
            r = ref[v, ch]
            g = got[v, ch].astype(np.float64)
            assert np.max(np.abs(g - r)) <= 1e-4 * np.max(np.abs(r))
            assert np.linalg.norm(g - r) <= 1e-4 * np.linalg.norm(r)


def _assert_batched_adjoint(got, ref, what):
    for v in range(ref.shape[0]):
        for ch in range(ref.shape[1]):
            r = ref[v, ch]
            g = got[v, ch].astype(np.float64)
            assert np.max(np.abs(g - r)) <= 1e-4 * np.max(np.abs(r)), f"{what} ({v}, {ch})"
            assert np.linalg.norm(g - r) <= 1e-4 * np.linalg.norm(r), f"{what} ({v}, {ch})"


# rays much closer than a voxel (as in the adjoint's record-path tests): with
# a workspace every image takes the record path of its volume-channel
DENSE = dict(dims=(23, 17, 29), H=150, W=170, n_samples=40)


@pytest.mark.parametrize("n_vols,C,n_views", [(2, 2, 4), (3, 1, 1)])
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
def test_batched_adjoint_with_workspace_dense_views(cuda, n_vols, C, n_views, mode):
    seed = 631 + n_views
    w = wl.small_random_case(seed, B=n_views, **DENSE)
    nx, ny, nz = w.dims
    vols = np.random.default_rng(seed).uniform(0.0, 0.05, (n_vols, C, nz, ny, nx)).astype(np.float32)
    n_out = n_vols if (n_views == 1 and n_vols > 1) else n_views
    go = np.random.default_rng(6).standard_normal((n_out, C, w.H, w.W)).astype(np.float32)
    fwd = _gpu_batched(w, vols, n_views, PADDED, mode) if mode else None
    ref = oracle.adjoint_batched(w.dims, w.spacing, w.origin, w.K, w.Rt, n_vols, n_views, w.H,
                                 w.W, w.n_samples, w.density_factor, mode, go, vols=vols,
                                 nthreads=8)
    for workspace in (False, True):
        got = _gpu_adjoint_batched(w, n_vols, C, n_views, go, mode, fwd, workspace=workspace)
        _assert_batched_adjoint(got, ref, f"workspace {workspace}")


def test_batched_adjoint_with_workspace_sparse_views(cuda):
    # the plan leaves these images on the direct path
    w, vols = _batch(2, 3, 4, 641)
    go = np.random.default_rng(7).standard_normal((4, 3, w.H, w.W)).astype(np.float32)
    ref = oracle.adjoint_batched(w.dims, w.spacing, w.origin, w.K, w.Rt, 2, 4, w.H, w.W,
                                 w.n_samples, w.density_factor, wl.MODE_RAW, go, vols=vols,
                                 nthreads=4)
    got = _gpu_adjoint_batched(w, 2, 3, 4, go, wl.MODE_RAW, workspace=True)
    _assert_batched_adjoint(got, ref, "sparse, workspace")


def test_batched_adjoint_slab_pass(cuda):
    # sparse images of 2 volumes x 3 channels, a call large enough (31e6
    # ray-samples) for the slab pass: 13 slabs of 3 cell layers, records per
    # volume-channel slot
    w = wl.small_random_case(642, B=4, dims=(300, 280, 40), H=160, W=170, n_samples=96)
    nx, ny, nz = w.dims
    vols = np.random.default_rng(642).uniform(0.0, 0.05, (2, 3, nz, ny, nx)).astype(np.float32)
    go = np.random.default_rng(8).standard_normal((4, 3, w.H, w.W)).astype(np.float32)
    ref = oracle.adjoint_batched(w.dims, w.spacing, w.origin, w.K, w.Rt, 2, 4, w.H, w.W,
                                 w.n_samples, w.density_factor, wl.MODE_RAW, go, vols=vols,
                                 nthreads=8)
    got = _gpu_adjoint_batched(w, 2, 3, 4, go, wl.MODE_RAW, workspace=True)
    _assert_batched_adjoint(got, ref, "sparse, slab pass")
    assert drr.drr_wait_timeouts() == 0


def test_batched_dot_product_identity(cuda):
    w, x = _batch(2, 2, 6, 621)
    y = np.random.default_rng(9).standard_normal((6, 2, w.H, w.W)).astype(np.float32)
    Ax = _gpu_batched(w, x, 6, LINEAR, wl.MODE_RAW).astype(np.float64)
    ATy = _gpu_adjoint_batched(w, 2, 2, 6, y, wl.MODE_RAW).astype(np.float64)
    lhs = float(np.sum(Ax * y.astype(np.float64)))
    rhs = float(np.sum(x.astype(np.float64) * ATy))
    assert abs(lhs - rhs) <= 1e-5 * np.linalg.norm(Ax) * np.linalg.norm(y.astype(np.float64))


def _prepared_batch(vols, dims, dtype, layout):
    import torch
    n_vols, C = vols.shape[:2]
    v32 = torch.from_numpy(np.ascontiguousarray(vols)).cuda()
    per = drr.drr_prepared_bytes(dims, dtype, layout)
    src = torch.empty(n_vols * C * per, dtype=torch.uint8, device="cuda")
    for s in range(n_vols * C):
        drr.drr_prepare_volume(v32.view(n_vols * C, -1)[s], dims, dtype, layout,
                               src[s * per:(s + 1) * per], per)
    return src


@pytest.mark.parametrize("n_vols,C,n_views,mode", [(2, 2, 4, wl.MODE_RAW),
                                                   (3, 2, 1, wl.MODE_BEER_LAMBERT),
                                                   (2, 1, 2, wl.MODE_ALPHA)])
@pytest.mark.parametrize("layout,dtype", [(CORNERS, F32), (QUADS, BF16)])
def test_batched_pose_gradient(cuda, n_vols, C, n_views, mode, layout, dtype):
    # (3, 2, 1): one pose broadcast to three volumes, six images add into it
    import torch
    w, vols = _batch(n_vols, C, n_views, 651 + n_views)
    n_out = n_vols if (n_views == 1 and n_vols > 1) else n_views
    go = np.random.default_rng(8).standard_normal((n_out, C, w.H, w.W)).astype(np.float32)
    ref_vols = bf16_values(vols) if dtype == BF16 else vols
    ref = oracle.pose_grad_batched(ref_vols, w.dims, w.spacing, w.origin, w.K, w.Rt, n_views, w.H,
                                   w.W, w.n_samples, w.density_factor, mode, go, nthreads=8)
    src = _prepared_batch(vols, w.dims, dtype, layout)
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    fo = None
    if mode != wl.MODE_RAW:
        fo = torch.full((n_out, C, w.H, w.W), float("nan"), device="cuda")
        drr.drr_render_batched(src, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt, n_vols, C,
                               n_views, w.H, w.W, w.n_samples, w.density_factor, mode, fo)
    g = torch.zeros((n_views, 12), device="cuda")
    drr.drr_render_pose_grad_batched(src, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt,
                                     n_vols, C, n_views, w.H, w.W, w.n_samples, w.density_factor,
                                     mode, torch.from_numpy(go).cuda(), fo, g)
    torch.cuda.synchronize()
    assert_pose_parity(g.cpu().numpy().reshape(-1, 3, 4), ref, 1e-4,
                       what=f"batched ({n_vols}, {C}, {n_views}) layout {layout} dtype {dtype}")


@pytest.mark.parametrize("n_vols,C,n_views", [(2, 2, 4), (3, 1, 1)])
@pytest.mark.parametrize("layout,dtype", [(CORNERS, BF16), (QUADS, F32)])
def test_batched_alpha_volume_gradient(cuda, n_vols, C, n_views, layout, dtype):
    # dense geometry: with a workspace the images take the alpha record path of
    # their volume-channel; without one, the direct path
    import torch
    seed = 661 + n_views
    w = wl.small_random_case(seed, B=n_views, **DENSE)
    w.density_factor = 25.0
    nx, ny, nz = w.dims
    vols = np.random.default_rng(seed).uniform(0.0, 0.05, (n_vols, C, nz, ny, nx)).astype(np.float32)
    n_out = n_vols if (n_views == 1 and n_vols > 1) else n_views
    go = np.random.default_rng(9).standard_normal((n_out, C, w.H, w.W)).astype(np.float32)
    ref_vols = bf16_values(vols) if dtype == BF16 else vols
    ref = oracle.adjoint_batched(w.dims, w.spacing, w.origin, w.K, w.Rt, n_vols, n_views, w.H,
                                 w.W, w.n_samples, w.density_factor, wl.MODE_ALPHA, go,
                                 vols=ref_vols, nthreads=8)
    src = _prepared_batch(vols, w.dims, dtype, layout)
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    fo = torch.full((n_out, C, w.H, w.W), float("nan"), device="cuda")
    drr.drr_render_batched(src, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt, n_vols, C,
                           n_views, w.H, w.W, w.n_samples, w.density_factor, wl.MODE_ALPHA, fo)
    go_d = torch.from_numpy(go).cuda()
    for workspace in (False, True):
        g = torch.zeros((n_vols, C, nz, ny, nx), device="cuda")
        ws = None
        if workspace:
            ws = torch.full((drr.drr_adjoint_batched_workspace_bytes(w.dims, n_vols, C, n_views),),
                            0x7F, dtype=torch.uint8, device="cuda")
        drr.drr_render_alpha_adjoint_batched(src, dtype, layout, w.dims, w.spacing, w.origin, w.K,
                                             Rt, n_vols, C, n_views, w.H, w.W, w.n_samples,
                                             w.density_factor, go_d, fo, g, ws)
        torch.cuda.synchronize()
        _assert_batched_adjoint(g.cpu().numpy(), ref, f"alpha workspace {workspace}")

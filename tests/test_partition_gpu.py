"""The multi-GPU partition's per-rank work on one GPU: every rank's share of
the detector rows (whole views and row blocks rendered through shifted
intrinsics) through the CUDA path, assembled in rank order, against the fp64
oracle for the whole job -- the forward image, and the volume gradient summed
over the ranks (what the all-reduce forms), with and without a workspace.
Tolerances: the parity tests' (forward 1e-4 normwise and per pixel above 1 %
of the maximum; adjoint 1e-4 normwise and relative L2)."""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import partition as P
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


# 3 views of 37 x 29 pixels with rays denser than the voxels, so that dense
# views take the record path of the workspace adjoint
CASE = dict(seed=61, dims=(23, 17, 29), B=3, H=37, W=29, n_samples=40)


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
def test_rank_shares_reassemble_the_whole_job(cuda, world, mode):
    from cone_beam_ct_b200 import drr
    torch = cuda
    w = wl.small_random_case(**CASE)
    K = np.asarray(w.K, np.float32)
    # denser rays: a longer focal length makes a pixel much narrower than a voxel
    K = K.copy().reshape(3, 3)
    K[0, 0] *= 6.0
    K[1, 1] *= 6.0
    w.K = K.reshape(-1)
    nx, ny, nz = w.dims
    vol = torch.from_numpy(w.vol).cuda()
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    go = np.random.default_rng(62).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    ref_img = oracle.render(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                            w.density_factor, mode)
    ref_grad = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                              w.density_factor, mode, go, vol=w.vol, nthreads=4)
    grads = {False: torch.zeros((nz, ny, nx), device="cuda"),
             True: torch.zeros((nz, ny, nx), device="cuda")}
    ws = torch.full((drr.drr_adjoint_workspace_bytes(w.dims, w.B),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    pieces = []
    for rank in range(world):
        part = P.Partition(w.B, w.H, w.W, world, rank)
        out = torch.full((max(1, part.rays),), float("nan"), device="cuda")
        P.render_partitioned(part, vol, drr.DRR_F32, drr.DRR_LAYOUT_LINEAR, w.dims, w.spacing,
                             w.origin, w.K, Rt, w.n_samples, w.density_factor, mode, out)
        pieces.append(out[:part.rays])
        g_local = torch.from_numpy(go.reshape(-1)[part.local_slice()].copy()).cuda()
        fwd = out if mode == wl.MODE_BEER_LAMBERT else None
        for with_ws in (False, True):
            P.adjoint_partitioned(part, w.dims, w.spacing, w.origin, w.K, Rt, w.n_samples,
                                  w.density_factor, mode, g_local, fwd, grads[with_ws],
                                  workspace=ws if with_ws else None, reduce=False)
    torch.cuda.synchronize()
    img = torch.cat(pieces).cpu().numpy().reshape(w.B, w.H, w.W)
    assert_parity(img, ref_img, 1e-4, what=f"forward over {world} ranks")
    for with_ws, g in grads.items():
        got = g.cpu().numpy().astype(np.float64)
        scale = np.max(np.abs(ref_grad))
        norm = np.max(np.abs(got - ref_grad)) / scale
        l2 = np.linalg.norm(got - ref_grad) / np.linalg.norm(ref_grad)
        assert norm <= 1e-4 and l2 <= 1e-4, (f"adjoint over {world} ranks, workspace {with_ws}: "
                                             f"normwise {norm:.3g}, L2 {l2:.3g}")

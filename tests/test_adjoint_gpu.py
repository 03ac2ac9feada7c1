"""GPU adjoint parity: the volume-gradient scatter against the fp64 oracle
adjoint, and the dot-product identity <A x, y> = <x, A^T y> (TorchTomo page,
"Discrete Adjoint and Learned Primal-Dual") between the GPU forward and the
GPU adjoint.

Tolerances.  No page fixes one for the adjoint; the bar of the forward
(1e-4) is kept, read for a scatter whose voxels sum many random-sign terms
(so per-voxel relative error is meaningless where they cancel): normwise
max |gpu - oracle| / max |oracle| <= 1e-4 and relative L2 error <= 1e-4.
Dot-product residual |<Ax, y> - <x, A^T y>| / (||Ax|| ||y||) <= 1e-5 (fp32
sums of up to ~10^9 terms; the oracle itself meets 1e-12, see the pins).
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import (BF16, CORNERS, F32, LINEAR, PADDED, QUADS, bf16_values,
                               gpu_adjoint, gpu_forward)

pytestmark = pytest.mark.gpu
TOL_ADJ, TOL_DOT = 1e-4, 1e-5


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def assert_adjoint_parity(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.max(np.abs(ref))
    assert scale > 0
    norm = np.max(np.abs(got - ref)) / scale
    l2 = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert norm <= TOL_ADJ and l2 <= TOL_ADJ, f"{what}: normwise {norm:.3g}, L2 {l2:.3g}"


def _oracle_adjoint(w, go, mode, nthreads=8):
    return oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                          w.density_factor, mode, go, vol=w.vol, nthreads=nthreads)


@pytest.mark.parametrize("seed", [201, 202, 203])
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
@pytest.mark.parametrize("workspace", [False, True])
def test_small_ragged_adjoint(cuda, seed, mode, workspace):
    w = wl.small_random_case(seed)
    go = np.random.default_rng(seed).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=PADDED, dtype=F32, mode=mode) if mode else None
    got = gpu_adjoint(w, go, mode=mode, fwd_out=fwd, workspace=workspace)
    assert_adjoint_parity(got, _oracle_adjoint(w, go, mode), what=f"seed {seed} mode {mode}")


# rays much closer than a voxel (a 16-pixel tile spans ~2.5 voxels): these
# views take the corner-record path of drr_render_adjoint_ws
DENSE = dict(dims=(23, 17, 29), H=150, W=170, n_samples=40)


@pytest.mark.parametrize("seed", [211, 212])
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
def test_dense_views_take_the_record_path(cuda, seed, mode):
    w = wl.small_random_case(seed, **DENSE)
    go = np.random.default_rng(seed).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=PADDED, dtype=F32, mode=mode) if mode else None
    ref = _oracle_adjoint(w, go, mode)
    for workspace in (False, True):
        got = gpu_adjoint(w, go, mode=mode, fwd_out=fwd, workspace=workspace)
        assert_adjoint_parity(got, ref, what=f"dense seed {seed} workspace {workspace}")


def _mixed_case(seed, n_samples=DENSE["n_samples"]):
    """DENSE geometry with its last view moved 4x farther: one call whose plan
    sends two views to the record path and one to the sparse side (the
    direct path; the slab pass once the call has 8 * 2^20 ray-samples)."""
    w = wl.small_random_case(seed, **dict(DENSE, n_samples=n_samples))
    Rt = w.Rt.copy()
    Rt[2, :, 3] *= 4.0
    w.Rt = Rt
    return w


@pytest.mark.parametrize("n_samples", [40, 120])
def test_mixed_dense_and_sparse_views_in_one_call(cuda, n_samples):
    # 40 samples: the sparse view on the direct path; 120 (9.2e6 ray-samples):
    # the slab pass, in the record area the dense views' scatter just read
    import torch
    from cone_beam_ct_b200 import drr
    w = _mixed_case(214, n_samples)
    go = np.random.default_rng(214).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    ref = _oracle_adjoint(w, go, wl.MODE_RAW)
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    nx, ny, nz = w.dims
    grad = torch.zeros((nz, ny, nx), dtype=torch.float32, device="cuda")
    ws = torch.full((drr.drr_adjoint_workspace_bytes(w.dims, w.B),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W, w.n_samples,
                              w.density_factor, wl.MODE_RAW, torch.from_numpy(go).cuda(), None,
                              grad, ws)
    torch.cuda.synchronize()
    # white-box: the plan's flags at the head of the workspace (bit 0: some
    # view dense, bit 1: some view sparse; then one per view)
    flags = ws[:4 * (1 + w.B)].cpu().numpy().view(np.int32)
    assert flags.tolist() == [3, 1, 1, 0]
    assert_adjoint_parity(grad.cpu().numpy(), ref, what="mixed dense and sparse views")


# A wide, flat volume: every view is sparse (rays ~4 voxels apart), and a
# cell layer's records (699^2 cells x 32 bytes) are so large that the
# workspace adjoint's slab pass takes several slabs of 3 layers (the last one
# ragged: 11 cell layers), with rays crossing slab boundaries at every
# angle.  3 x 200 x 210 rays x 211 samples (26.6e6) is above the size below
# which a call sends its sparse views to the direct path instead.
WIDE_FLAT = dict(dims=(700, 700, 12), spacing=(1.0, 1.1, 0.9), H=200, W=210, n_samples=211)


@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
def test_sparse_views_take_the_slab_records(cuda, mode):
    import torch
    from cone_beam_ct_b200 import drr
    w = wl.small_random_case(216, **WIDE_FLAT)
    go = np.random.default_rng(216).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=PADDED, dtype=F32, mode=mode) if mode else None
    ref = _oracle_adjoint(w, go, mode)
    got = gpu_adjoint(w, go, mode=mode, fwd_out=fwd, workspace=True)
    assert_adjoint_parity(got, ref, what=f"slab records, mode {mode}")
    # the plan sent every view to the sparse side
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    nx, ny, nz = w.dims
    grad = torch.zeros((nz, ny, nx), dtype=torch.float32, device="cuda")
    ws = torch.full((drr.drr_adjoint_workspace_bytes(w.dims, w.B),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W, w.n_samples,
                              w.density_factor, wl.MODE_RAW, torch.from_numpy(go).cuda(), None,
                              grad, ws)
    torch.cuda.synchronize()
    assert ws[:4 * (1 + w.B)].cpu().numpy().view(np.int32).tolist() == [2] + [0] * w.B
    # no grid-barrier wait of the slab pass gave up
    assert drr.drr_wait_timeouts() == 0


@pytest.mark.parametrize("nz", [2, 3])
def test_slab_pass_on_one_or_two_cell_layers(cuda, nz):
    # the degenerate depths: one cell layer (nz = 2) and two (nz = 3), one
    # slab either way, every ray crossing the whole depth in a few samples
    w = wl.small_random_case(217 + nz, dims=(400, 380, nz), B=2, H=256, W=256, n_samples=80)
    assert w.B * w.H * w.W * w.n_samples >= 8 * 2 ** 20       # the slab pass's size
    go = np.random.default_rng(nz).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    ref = _oracle_adjoint(w, go, wl.MODE_RAW)
    import torch
    from cone_beam_ct_b200 import drr
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    nx, ny, _ = w.dims
    grad = torch.zeros((nz, ny, nx), dtype=torch.float32, device="cuda")
    ws = torch.full((drr.drr_adjoint_workspace_bytes(w.dims, w.B),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W, w.n_samples,
                              w.density_factor, wl.MODE_RAW, torch.from_numpy(go).cuda(), None,
                              grad, ws)
    torch.cuda.synchronize()
    assert ws[:4 * (1 + w.B)].cpu().numpy().view(np.int32).tolist() == [2] + [0] * w.B
    assert_adjoint_parity(grad.cpu().numpy(), ref, what=f"slab pass, nz = {nz}")


def test_record_path_dot_product_identity(cuda):
    w = wl.small_random_case(213, **DENSE)
    rng = np.random.default_rng(7)
    nx, ny, nz = w.dims
    x = rng.uniform(0, 1, (nz, ny, nx)).astype(np.float32)
    y = rng.standard_normal((w.B, w.H, w.W)).astype(np.float32)
    Ax = gpu_forward(w, layout=LINEAR, dtype=F32, mode=wl.MODE_RAW, vol=x).astype(np.float64)
    ATy = gpu_adjoint(w, y, mode=wl.MODE_RAW, workspace=True).astype(np.float64)
    lhs = float(np.dot(Ax.reshape(-1), y.reshape(-1).astype(np.float64)))
    rhs = float(np.dot(x.reshape(-1).astype(np.float64), ATy.reshape(-1)))
    assert abs(lhs - rhs) / (np.linalg.norm(Ax) * np.linalg.norm(y.astype(np.float64))) <= TOL_DOT


def _dot_residual(w, x, y, layout, workspace=False):
    Ax = gpu_forward(w, layout=layout, dtype=F32, mode=wl.MODE_RAW, vol=x).astype(np.float64)
    ATy = gpu_adjoint(w, y, mode=wl.MODE_RAW, workspace=workspace).astype(np.float64)
    lhs = float(np.dot(Ax.reshape(-1), y.reshape(-1).astype(np.float64)))
    rhs = float(np.dot(x.reshape(-1).astype(np.float64), ATy.reshape(-1)))
    return abs(lhs - rhs) / (np.linalg.norm(Ax) * np.linalg.norm(y.astype(np.float64)))


@pytest.mark.parametrize("layout", [LINEAR, PADDED])
def test_dot_product_identity_small(cuda, layout):
    w = wl.small_random_case(204)
    rng = np.random.default_rng(5)
    nx, ny, nz = w.dims
    x = rng.uniform(0, 1, (nz, ny, nx)).astype(np.float32)
    y = rng.standard_normal((w.B, w.H, w.W)).astype(np.float32)
    assert _dot_residual(w, x, y, layout) <= TOL_DOT


def test_adjoint_accumulates_and_skips_zero_gradient(cuda):
    import torch
    from cone_beam_ct_b200 import drr
    w = wl.small_random_case(205)
    go = np.random.default_rng(1).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    once = gpu_adjoint(w, go, mode=wl.MODE_RAW)
    Rt = torch.from_numpy(w.Rt.reshape(-1, 12).copy()).cuda()
    g = torch.from_numpy(once).cuda()
    drr.drr_render_adjoint(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W, w.n_samples,
                           w.density_factor, wl.MODE_RAW, torch.from_numpy(go).cuda(), None, g)
    torch.cuda.synchronize()
    assert np.allclose(g.cpu().numpy(), 2 * once, rtol=1e-5, atol=1e-6 * np.abs(once).max())
    zero = gpu_adjoint(w, np.zeros_like(go), mode=wl.MODE_RAW)
    assert np.all(zero == 0.0)


@pytest.mark.slow
def test_config5_full_adjoint_and_dot_product(cuda):
    w = wl.make_config(5)
    ref = _oracle_adjoint(w, w.grad_out, w.mode, nthreads=16)
    for workspace in (False, True):
        got = gpu_adjoint(w, w.grad_out, mode=w.mode, workspace=workspace)
        assert_adjoint_parity(got, ref, what=f"config 5 workspace {workspace}")
    rng = np.random.default_rng(55)
    nx, ny, nz = w.dims
    x = rng.uniform(0, 1, (nz, ny, nx)).astype(np.float32)
    y = rng.standard_normal((w.B, w.H, w.W)).astype(np.float32)
    assert _dot_residual(w, x, y, PADDED) <= TOL_DOT


@pytest.mark.slow
def test_config2_full_adjoint_as_timed(cuda):
    # the 64-view workload's adjoint as the throughput run's configs block
    # times it: Beer-Lambert, a dense N(0, 1) upstream gradient, fwd_out from
    # the GPU forward in the xy-quad layout, a workspace (every view sparse:
    # the slab pass, 11 slabs), against the oracle on the whole volume
    w = wl.make_config(2)
    go = np.random.default_rng(2002).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=QUADS, dtype=F32, mode=wl.MODE_BEER_LAMBERT)
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, wl.MODE_BEER_LAMBERT, go, vol=w.vol, nthreads=16)
    got = gpu_adjoint(w, go, mode=wl.MODE_BEER_LAMBERT, fwd_out=fwd, workspace=True)
    assert_adjoint_parity(got, ref, what="config 2, Beer-Lambert, workspace")


@pytest.mark.slow
def test_config4_dense_band_adjoint(cuda):
    # the 512^3 volume seen by 2 C-arm views of 2048^2 with 256 samples, raw:
    # its record array (4.3 GB) is past 1 GiB, where the record kernel spreads
    # its warp phases over the first quarter of each ray; a band of 40 full
    # detector rows per view carries a dense N(0, 1) upstream gradient
    w = wl.make_config(4)
    go = np.zeros((w.B, w.H, w.W), np.float32)
    go[:, 1004:1044, :] = np.random.default_rng(44).standard_normal(
        (w.B, 40, w.W)).astype(np.float32)
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, wl.MODE_RAW, go, nthreads=16)
    got = gpu_adjoint(w, go, mode=wl.MODE_RAW, workspace=True)
    assert_adjoint_parity(got, ref, what="config 4 dense band")


@pytest.mark.slow
def test_config3_geometry_adjoint(cuda):
    # the 1024^2 x 512 C-arm geometry with an fp32 gradient volume: the dot-product
    # identity at full size, and the oracle on a sparse upstream gradient (2000 rays)
    w = wl.make_config(3)
    rng = np.random.default_rng(33)
    nx, ny, nz = w.dims
    x = rng.uniform(0, 1, (nz, ny, nx)).astype(np.float32)
    y = rng.standard_normal((w.B, w.H, w.W)).astype(np.float32)
    assert _dot_residual(w, x, y, PADDED) <= TOL_DOT
    assert _dot_residual(w, x, y, PADDED, workspace=True) <= TOL_DOT
    sparse = np.zeros((w.B, w.H, w.W), np.float32)
    ids = rng.choice(w.rays, size=2000, replace=False)
    sparse.reshape(-1)[ids] = rng.standard_normal(2000).astype(np.float32)
    ref = _oracle_adjoint(w, sparse, wl.MODE_RAW)
    for workspace in (False, True):
        got = gpu_adjoint(w, sparse, mode=wl.MODE_RAW, workspace=workspace)
        assert_adjoint_parity(got, ref, what=f"config 3 sparse upstream, workspace {workspace}")


# A contiguous band of full detector rows at the 1024^2 x 512 C-arm geometry:
# rows 472-567 of every view, so the band covers whole 32-row tiles of the
# dense-view path and ragged ones at both ends, with every ray of it live.
BAND_ROWS = slice(472, 568)


def dense_band(w, seed):
    go = np.zeros((w.B, w.H, w.W), np.float32)
    rng = np.random.default_rng(seed)
    n = BAND_ROWS.stop - BAND_ROWS.start
    go[:, BAND_ROWS, :] = rng.standard_normal((w.B, n, w.W)).astype(np.float32)
    return go


@pytest.mark.slow
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
def test_config3_dense_band_adjoint_as_timed(cuda, mode):
    # the adjoint the throughput run times: 256^3 volume (bf16 corner records
    # for the forward), 4 C-arm views of 1024^2, 512 samples, a dense N(0, 1)
    # upstream gradient, drr_render_adjoint_ws; in Beer-Lambert mode fwd_out
    # comes from the GPU forward and the oracle recomputes exp(-I) from the
    # same bf16-rounded volume
    w = wl.make_config(3)
    go = dense_band(w, 330 + mode)
    vb = bf16_values(w.vol)
    fwd = gpu_forward(w, layout=CORNERS, dtype=BF16, mode=mode) if mode else None
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, mode, go, vol=vb, nthreads=4)
    got = gpu_adjoint(w, go, mode=mode, fwd_out=fwd, workspace=True)
    assert_adjoint_parity(got, ref, what=f"config 3 dense band, mode {mode}")

"""The allocation-free adjoint (drr_render_adjoint_noalloc), for callers that
may not allocate device memory -- code under a memory manager that owns the
whole device, or a real-time loop where an allocation could synchronise the
device.  Its workspace is the library's built-in 32 MiB scratch, shared by
every call.

Each case runs the call twice in a row (the scratch keeps the previous
call's contents, so the second call shows that each call re-initialises
what it reads) and checks both results against the fp64 oracle's adjoint
and against the ordinary workspace adjoint (drr_render_adjoint_ws), in the
raw and the Beer-Lambert mode (where fwd_out, from the GPU forward, is
read).  Tolerance: the other adjoint tests' (normwise max error and relative
L2 error, each <= 1e-4).  This file is collected last so that a failure here
leaves every other test already run; it also passes on its own in a fresh
process."""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import F32, PADDED, gpu_forward

pytestmark = pytest.mark.gpu
TOL_ADJ = 1e-4


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from cone_beam_ct_b200 import drr
    drr.lib()
    return torch


def _inputs(torch, w, seed, mode):
    go = np.random.default_rng(seed).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    fwd = gpu_forward(w, layout=PADDED, dtype=F32, mode=mode) if mode else None
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return dev(w.Rt.reshape(-1, 12)), dev(go), dev(fwd), go


def _adjoint(torch, w, Rt, go, fwd, mode, noalloc):
    from cone_beam_ct_b200 import drr
    nx, ny, nz = w.dims
    grad = torch.zeros((nz, ny, nx), dtype=torch.float32, device="cuda")
    if noalloc:
        drr.drr_render_adjoint_noalloc(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
                                       w.n_samples, w.density_factor, mode, go, fwd, grad)
    else:
        nbytes = drr.drr_adjoint_workspace_bytes(w.dims, w.B)
        ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
        drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
                                  w.n_samples, w.density_factor, mode, go, fwd, grad, ws)
    torch.cuda.synchronize()
    return grad.cpu().numpy().astype(np.float64)


def _close(got, ref, what):
    scale = np.max(np.abs(ref))
    assert scale > 0
    norm = np.max(np.abs(got - ref)) / scale
    l2 = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert norm <= TOL_ADJ and l2 <= TOL_ADJ, f"{what}: normwise {norm:.3g}, L2 {l2:.3g}"


# dense views (rays much closer than a voxel) use the scratch's corner records;
# the sparse views of a small call use it only for the view flags, those of a
# call of at least 8 * 2^20 ray-samples for the slab pass's records
CASES = {
    "dense": dict(seed=301, dims=(23, 17, 29), H=150, W=170, n_samples=40),
    "dense, near the size limit": dict(seed=302, dims=(96, 96, 90), B=2, H=400, W=400,
                                        n_samples=64),
    "sparse": dict(seed=303),
    "sparse, slab pass": dict(seed=305, dims=(90, 84, 88), B=3, H=150, W=150, n_samples=160),
}


@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_the_oracle_and_the_workspace_adjoint_twice_in_a_row(cuda, name, mode):
    from cone_beam_ct_b200 import drr
    w = wl.small_random_case(**CASES[name])
    assert drr.drr_adjoint_workspace_bytes(w.dims, w.B) <= drr.DRR_NOALLOC_SCRATCH_BYTES
    Rt, go, fwd, go_host = _inputs(cuda, w, 7, mode)
    ref = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                         w.density_factor, mode, go_host, vol=w.vol, nthreads=8)
    with_ws = _adjoint(cuda, w, Rt, go, fwd, mode, noalloc=False)
    _close(with_ws, ref, f"{name}, mode {mode}, workspace adjoint against the oracle")
    for call in (1, 2):
        got = _adjoint(cuda, w, Rt, go, fwd, mode, noalloc=True)
        _close(got, ref, f"{name}, mode {mode}, call {call} against the oracle")
        _close(got, with_ws, f"{name}, mode {mode}, call {call} against the workspace adjoint")


def test_the_slab_case_is_all_sparse(cuda):
    # white-box: the plan sends every view of that case to the sparse side
    from cone_beam_ct_b200 import drr
    w = wl.small_random_case(**CASES["sparse, slab pass"])
    Rt, go, _, _ = _inputs(cuda, w, 7, wl.MODE_RAW)
    nx, ny, nz = w.dims
    grad = cuda.zeros((nz, ny, nx), dtype=cuda.float32, device="cuda")
    ws = cuda.full((drr.drr_adjoint_workspace_bytes(w.dims, w.B),), 0x7F, dtype=cuda.uint8,
                   device="cuda")
    drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W, w.n_samples,
                              w.density_factor, wl.MODE_RAW, go, None, grad, ws)
    cuda.cuda.synchronize()
    assert ws[:4 * (1 + w.B)].cpu().numpy().view(np.int32).tolist() == [2] + [0] * w.B


def test_noalloc_rejects_volumes_beyond_its_scratch(cuda):
    from cone_beam_ct_b200 import drr
    w = wl.small_random_case(304, dims=(128, 128, 128))
    assert drr.drr_adjoint_workspace_bytes(w.dims, w.B) > drr.DRR_NOALLOC_SCRATCH_BYTES
    Rt, go, _, _ = _inputs(cuda, w, 8, wl.MODE_RAW)
    nx, ny, nz = w.dims
    grad = cuda.zeros((nz, ny, nx), dtype=cuda.float32, device="cuda")
    with pytest.raises(drr.DrrError) as e:
        drr.drr_render_adjoint_noalloc(w.dims, w.spacing, w.origin, w.K, Rt, w.B, w.H, w.W,
                                       w.n_samples, w.density_factor, wl.MODE_RAW, go, None,
                                       grad)
    assert e.value.status == drr.DRR_ERR_UNSUPPORTED
    assert "built-in scratch" in drr.drr_get_last_error()
    cuda.cuda.synchronize()
    assert cuda.count_nonzero(grad).item() == 0

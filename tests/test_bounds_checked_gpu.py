"""The bounds-checked debug build (libdrr_checked.so, include/drr_debug.h):
every gather and scatter of every kernel range-checked against the extent
of its buffer.  Small ragged cases run through every entry point and layout
on it -- forward (4 layouts x fp32/bf16 x raw/Beer-Lambert/alpha), volume
adjoint (direct and with a workspace, sparse and dense views, the slab pass
of large sparse calls), pose gradient,
alpha gradient, Siddon pair, batches, prepare -- and the device error word
must stay 0: no index of any kernel leaves its buffer.  The results must also
match the ordinary build's (same arithmetic; the checks only guard)."""
import numpy as np
import pytest

from cone_beam_ct_b200 import workloads as wl
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def checked():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from cone_beam_ct_b200 import drr
    previous = drr.use_library(drr.CHECKED_LIB_PATH)
    drr.lib()
    drr.drr_debug_bounds_errors()               # start from a clean word
    yield drr
    drr.use_library(previous)


def _clean(drr, what):
    import torch
    torch.cuda.synchronize()
    count, first = drr.drr_debug_bounds_errors()
    assert count == 0, f"{what}: {count} out-of-range accesses (first at element {first})"


CASES = [dict(seed=501), dict(seed=502, dims=(23, 17, 29), H=150, W=170, n_samples=40),
         dict(seed=503, dims=(7, 5, 9), B=2, H=13, W=11, n_samples=5)]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_forward_every_layout_dtype_and_mode_stays_in_bounds(checked, case):
    w = wl.small_random_case(**CASES[case])
    for layout in H.LAYOUTS:
        for dtype in (H.F32, H.BF16):
            for mode in (wl.MODE_RAW, wl.MODE_BEER_LAMBERT, wl.MODE_ALPHA):
                H.gpu_forward(w, layout=layout, dtype=dtype, mode=mode)
                _clean(checked, f"forward layout {layout} dtype {dtype} mode {mode}")
    for dtype in (H.F32, H.BF16):
        for mode in (wl.MODE_RAW, wl.MODE_BEER_LAMBERT):
            H.gpu_forward_staged(w, dtype=dtype, mode=mode)
            _clean(checked, f"staged bricked forward dtype {dtype} mode {mode}")


@pytest.mark.parametrize("case", range(len(CASES)))
def test_adjoints_and_pose_gradient_stay_in_bounds(checked, case):
    w = wl.small_random_case(**CASES[case])
    go = np.random.default_rng(7).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    for mode in (wl.MODE_RAW, wl.MODE_BEER_LAMBERT):
        fwd = H.gpu_forward(w, layout=H.PADDED, dtype=H.F32, mode=mode)
        for workspace in (False, True):
            H.gpu_adjoint(w, go, mode=mode, fwd_out=fwd, workspace=workspace)
            _clean(checked, f"adjoint mode {mode} workspace {workspace}")
        if checked.drr_adjoint_workspace_bytes(w.dims, w.B) <= checked.DRR_NOALLOC_SCRATCH_BYTES:
            import torch
            nx, ny, nz = w.dims
            grad = torch.zeros((nz, ny, nx), device="cuda")
            checked.drr_render_adjoint_noalloc(
                w.dims, w.spacing, w.origin, w.K,
                torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda(), w.B, w.H,
                w.W, w.n_samples, w.density_factor, mode, torch.from_numpy(go).cuda(),
                torch.from_numpy(fwd).cuda() if mode else None, grad)
            _clean(checked, f"allocation-free adjoint mode {mode}")
        for layout in H.LAYOUTS:
            for dtype in (H.F32, H.BF16):
                H.gpu_pose_grad(w, go, layout=layout, dtype=dtype, mode=mode, fwd_out=fwd)
                _clean(checked, f"pose gradient layout {layout} dtype {dtype} mode {mode}")
    alpha = H.gpu_forward(w, layout=H.LINEAR, dtype=H.F32, mode=wl.MODE_ALPHA)
    for layout in (H.LINEAR, H.CORNERS, H.QUADS, H.BRICKS):
        for workspace in (False, True):
            H.gpu_alpha_adjoint(w, go, alpha, layout=layout, dtype=H.F32, workspace=workspace)
            _clean(checked, f"alpha adjoint layout {layout} workspace {workspace}")
    H.gpu_pose_grad(w, go, layout=H.CORNERS, dtype=H.F32, mode=wl.MODE_ALPHA, fwd_out=alpha)
    _clean(checked, "alpha pose gradient")
    H.gpu_siddon(w, mode=wl.MODE_RAW)
    H.gpu_siddon_adjoint(w, go, mode=wl.MODE_RAW)
    _clean(checked, "Siddon pair")


def test_batches_stay_in_bounds(checked):
    import torch
    drr = checked
    w = wl.small_random_case(504, dims=(19, 21, 17), B=6, H=40, W=36, n_samples=24)
    n_vols, channels = 3, 2
    nx, ny, nz = w.dims
    vols32 = np.stack([w.vol * (1 + 0.1 * v) for v in range(n_vols * channels)]).astype(np.float32)
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    for layout in H.LAYOUTS:
        per = drr.drr_prepared_bytes(w.dims, drr.DRR_F32, layout)
        vols = torch.empty(n_vols * channels * per, dtype=torch.uint8, device="cuda")
        for v in range(n_vols * channels):
            drr.drr_prepare_volume(torch.from_numpy(vols32[v]).cuda(), w.dims, drr.DRR_F32,
                                   layout, vols[v * per:(v + 1) * per], per)
        for n_views in (1, w.B):
            n_out = n_vols if n_views == 1 else n_views
            out = torch.empty((n_out, channels, w.H, w.W), device="cuda")
            drr.drr_render_batched(vols, drr.DRR_F32, layout, w.dims, w.spacing, w.origin, w.K,
                                   Rt[:n_views], n_vols, channels, n_views, w.H, w.W,
                                   w.n_samples, w.density_factor, wl.MODE_BEER_LAMBERT, out)
            go = torch.randn((n_out, channels, w.H, w.W), device="cuda")
            grads = torch.zeros((n_vols, channels, nz, ny, nx), device="cuda")
            ws = torch.empty(drr.drr_adjoint_batched_workspace_bytes(w.dims, n_vols, channels,
                                                                     n_views),
                             dtype=torch.uint8, device="cuda")
            drr.drr_render_adjoint_batched_ws(w.dims, w.spacing, w.origin, w.K, Rt[:n_views],
                                              n_vols, channels, n_views, w.H, w.W, w.n_samples,
                                              w.density_factor, wl.MODE_BEER_LAMBERT, go, out,
                                              grads, ws)
            g_rt = torch.zeros((n_views, 12), device="cuda")
            drr.drr_render_pose_grad_batched(vols, drr.DRR_F32, layout, w.dims, w.spacing,
                                             w.origin, w.K, Rt[:n_views], n_vols, channels,
                                             n_views, w.H, w.W, w.n_samples, w.density_factor,
                                             wl.MODE_BEER_LAMBERT, go, out, g_rt)
            _clean(drr, f"batches, layout {layout}, {n_views} views")


def test_slab_pass_stays_in_bounds(checked):
    # sparse views in a call large enough for the adjoint's slab pass (26.6e6
    # ray-samples, 4 slabs of 3 cell layers over a wide, flat volume)
    w = wl.small_random_case(506, dims=(700, 700, 12), spacing=(1.0, 1.1, 0.9), H=200, W=210,
                             n_samples=211)
    go = np.random.default_rng(9).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    for mode in (wl.MODE_RAW, wl.MODE_BEER_LAMBERT):
        fwd = H.gpu_forward(w, layout=H.PADDED, dtype=H.F32, mode=mode) if mode else None
        H.gpu_adjoint(w, go, mode=mode, fwd_out=fwd, workspace=True)
        _clean(checked, f"slab pass mode {mode}")
    assert checked.drr_wait_timeouts() == 0


def test_checked_results_match_the_ordinary_build(checked):
    drr = checked
    w = wl.small_random_case(505)
    go = np.random.default_rng(8).standard_normal((w.B, w.H, w.W)).astype(np.float32)
    got = (H.gpu_forward(w, layout=H.CORNERS, dtype=H.BF16),
           H.gpu_adjoint(w, go, mode=wl.MODE_RAW, workspace=True))
    _clean(drr, "forward and adjoint")
    previous = drr.use_library(drr.LIB_PATH.replace("libdrr_checked.so", "libdrr.so"))
    try:
        ref = (H.gpu_forward(w, layout=H.CORNERS, dtype=H.BF16),
               H.gpu_adjoint(w, go, mode=wl.MODE_RAW, workspace=True))
    finally:
        drr.use_library(previous)
    assert np.array_equal(got[0], ref[0])
    scale = np.max(np.abs(ref[1]))
    assert np.max(np.abs(got[1] - ref[1])) <= 1e-6 * scale     # atomics: order may differ

"""Helpers of the GPU parity tests: run the CUDA path through the C ABI
(cone_beam_ct_b200.drr) on a Workload, and compare against the oracle with
the tolerances the tests state."""
import numpy as np

from cone_beam_ct_b200 import drr

LINEAR, PADDED, CORNERS = drr.DRR_LAYOUT_LINEAR, drr.DRR_LAYOUT_PADDED, drr.DRR_LAYOUT_CORNERS
QUADS, BRICKS = drr.DRR_LAYOUT_QUADS, drr.DRR_LAYOUT_BRICKS
LAYOUTS = (LINEAR, PADDED, CORNERS, QUADS, BRICKS)
F32, BF16 = drr.DRR_F32, drr.DRR_BF16


def device_inputs(w, vol=None):
    import torch
    v = torch.from_numpy(np.ascontiguousarray(w.vol if vol is None else vol)).cuda()
    Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12))).cuda()
    return v, Rt


def prepared(vol32, dims, dtype, layout):
    """The volume in the layout/dtype drr_render reads (prepared on the GPU)."""
    import torch
    if dtype == F32 and layout == LINEAR:
        return vol32
    nbytes = drr.drr_prepared_bytes(dims, dtype, layout)
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    drr.drr_prepare_volume(vol32, dims, dtype, layout, buf)
    return buf


def gpu_forward(w, layout=PADDED, dtype=None, mode=None, vol=None, Rt=None):
    import torch
    dtype = w.dtype if dtype is None else dtype
    mode = w.mode if mode is None else mode
    v32, Rt_d = device_inputs(w, vol)
    if Rt is not None:
        Rt_d = torch.from_numpy(np.ascontiguousarray(Rt.reshape(-1, 12), dtype=np.float32)).cuda()
    B = Rt_d.shape[0]
    src = prepared(v32, w.dims, dtype, layout)
    out = torch.full((B, w.H, w.W), float("nan"), dtype=torch.float32, device="cuda")
    drr.drr_render(src, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt_d, B, w.H, w.W,
                   w.n_samples, w.density_factor, mode, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def gpu_forward_staged(w, dtype=None, mode=None):
    """drr_render_staged: the bricked forward with each frustum layer staged in
    shared memory."""
    import torch
    dtype = w.dtype if dtype is None else dtype
    mode = w.mode if mode is None else mode
    v32, Rt_d = device_inputs(w)
    src = prepared(v32, w.dims, dtype, BRICKS)
    out = torch.full((w.B, w.H, w.W), float("nan"), dtype=torch.float32, device="cuda")
    drr.drr_render_staged(src, dtype, w.dims, w.spacing, w.origin, w.K, Rt_d, w.B, w.H, w.W,
                          w.n_samples, w.density_factor, mode, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def gpu_adjoint(w, grad_out, mode=None, fwd_out=None, workspace=False):
    """Volume gradient through drr_render_adjoint, or drr_render_adjoint_ws
    with a fresh workspace (filled with garbage first: its content on entry
    must not matter)."""
    import torch
    mode = w.mode if mode is None else mode
    _, Rt_d = device_inputs(w, vol=np.zeros((1,), np.float32))
    go = torch.from_numpy(np.ascontiguousarray(grad_out, dtype=np.float32)).cuda()
    fo = None
    if fwd_out is not None:
        fo = torch.from_numpy(np.ascontiguousarray(fwd_out, dtype=np.float32)).cuda()
    nx, ny, nz = w.dims
    grad = torch.zeros((nz, ny, nx), dtype=torch.float32, device="cuda")
    if workspace:
        nbytes = drr.drr_adjoint_workspace_bytes(w.dims, w.B)
        ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
        drr.drr_render_adjoint_ws(w.dims, w.spacing, w.origin, w.K, Rt_d, w.B, w.H, w.W,
                                  w.n_samples, w.density_factor, mode, go, fo, grad, ws)
    else:
        drr.drr_render_adjoint(w.dims, w.spacing, w.origin, w.K, Rt_d, w.B, w.H, w.W,
                               w.n_samples, w.density_factor, mode, go, fo, grad)
    torch.cuda.synchronize()
    return grad.cpu().numpy()


def bf16_values(vol):
    """The volume as bf16-rounded fp32 values (oracle-side rounding)."""
    import oracle
    return oracle.bf16_to_float(oracle.round_bf16(vol))


def parity_errors(got, ref, floor=1e-2):
    """(normwise max error / max|ref|, worst per-element relative error over
    elements with |ref| >= floor * max|ref|)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    scale = float(np.max(np.abs(ref)))
    if scale == 0.0:
        return float(np.max(np.abs(got))), 0.0
    diff = np.abs(got - ref)
    big = np.abs(ref) >= floor * scale
    rel = float(np.max(diff[big] / np.abs(ref[big]))) if np.any(big) else 0.0
    return float(np.max(diff)) / scale, rel


def assert_parity(got, ref, tol, floor=1e-2, what=""):
    norm, rel = parity_errors(got, ref, floor)
    assert norm <= tol and rel <= tol, f"{what}: normwise {norm:.3g}, per-element {rel:.3g} > {tol}"
    return norm, rel


def gpu_pose_grad(w, grad_out, layout=LINEAR, dtype=F32, mode=None, fwd_out=None, accumulate=None):
    """dL/d[R|t] (B x 3 x 4) through drr_render_pose_grad; ``accumulate`` is an
    initial value of grad_Rt (zeros by default)."""
    import torch
    mode = w.mode if mode is None else mode
    v32, Rt_d = device_inputs(w)
    src = prepared(v32, w.dims, dtype, layout)
    go = torch.from_numpy(np.ascontiguousarray(grad_out, dtype=np.float32)).cuda()
    fo = None
    if fwd_out is not None:
        fo = torch.from_numpy(np.ascontiguousarray(fwd_out, dtype=np.float32)).cuda()
    init = np.zeros((w.B, 12), np.float32) if accumulate is None else accumulate.reshape(w.B, 12)
    g = torch.from_numpy(np.ascontiguousarray(init, dtype=np.float32)).cuda()
    drr.drr_render_pose_grad(src, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt_d, w.B,
                             w.H, w.W, w.n_samples, w.density_factor, mode, go, fo, g)
    torch.cuda.synchronize()
    return g.cpu().numpy().reshape(w.B, 3, 4)


def assert_pose_parity(got, ref, tol, what=""):
    """Per view, the rotation block and the translation column (different
    units) each within tol of the oracle, normwise: max|got - ref| / max|ref|."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite pose gradient"
    worst = 0.0
    for b in range(ref.shape[0]):
        for sl in (np.s_[:, :3], np.s_[:, 3]):
            scale = np.max(np.abs(ref[b][sl]))
            err = np.max(np.abs(got[b][sl] - ref[b][sl])) / scale if scale > 0 else np.max(
                np.abs(got[b][sl]))
            worst = max(worst, err)
    assert worst <= tol, f"{what}: pose gradient normwise error {worst:.3g} > {tol}"
    return worst


def gpu_alpha_adjoint(w, grad_out, fwd_out, layout=LINEAR, dtype=F32, workspace=False):
    """Volume gradient of the alpha image through drr_render_alpha_adjoint, or
    drr_render_alpha_adjoint_ws with a fresh workspace filled with garbage."""
    import torch
    v32, Rt_d = device_inputs(w)
    src = prepared(v32, w.dims, dtype, layout)
    go = torch.from_numpy(np.ascontiguousarray(grad_out, dtype=np.float32)).cuda()
    fo = torch.from_numpy(np.ascontiguousarray(fwd_out, dtype=np.float32)).cuda()
    nx, ny, nz = w.dims
    grad = torch.zeros((nz, ny, nx), dtype=torch.float32, device="cuda")
    if workspace:
        nbytes = drr.drr_adjoint_workspace_bytes(w.dims, w.B)
        ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
        drr.drr_render_alpha_adjoint_ws(src, dtype, layout, w.dims, w.spacing, w.origin, w.K,
                                        Rt_d, w.B, w.H, w.W, w.n_samples, w.density_factor, go,
                                        fo, grad, ws)
    else:
        drr.drr_render_alpha_adjoint(src, dtype, layout, w.dims, w.spacing, w.origin, w.K, Rt_d,
                                     w.B, w.H, w.W, w.n_samples, w.density_factor, go, fo, grad)
    torch.cuda.synchronize()
    return grad.cpu().numpy()


def gpu_siddon(w, dtype=F32, mode=None, vol=None):
    """Cell-constant image through drr_render_siddon (linear volume)."""
    import torch
    mode = w.mode if mode is None else mode
    v32, Rt_d = device_inputs(w, vol)
    src = prepared(v32, w.dims, dtype, LINEAR)
    out = torch.full((w.B, w.H, w.W), float("nan"), dtype=torch.float32, device="cuda")
    drr.drr_render_siddon(src, dtype, w.dims, w.spacing, w.origin, w.K, Rt_d, w.B, w.H, w.W,
                          w.density_factor, mode, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def gpu_siddon_adjoint(w, grad_out, mode=None, fwd_out=None):
    import torch
    mode = w.mode if mode is None else mode
    _, Rt_d = device_inputs(w, vol=np.zeros((1,), np.float32))
    go = torch.from_numpy(np.ascontiguousarray(grad_out, dtype=np.float32)).cuda()
    fo = None
    if fwd_out is not None:
        fo = torch.from_numpy(np.ascontiguousarray(fwd_out, dtype=np.float32)).cuda()
    nx, ny, nz = w.dims
    grad = torch.zeros((nz, ny, nx), dtype=torch.float32, device="cuda")
    drr.drr_render_siddon_adjoint(w.dims, w.spacing, w.origin, w.K, Rt_d, w.B, w.H, w.W,
                                  w.density_factor, mode, go, fo, grad)
    torch.cuda.synchronize()
    return grad.cpu().numpy()

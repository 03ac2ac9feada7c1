"""The largest volumes the ABI accepts, for each layout: the 32-bit element
and cell index arithmetic of the kernels at its top end.

Inputs are made on the GPU (no host copy of multi-GB arrays) and checked
against closed forms, not the oracle: an affine volume v = a + b i + c j + d k
is reproduced exactly by trilinear interpolation inside the voxel-centre box,
and the midpoint rule integrates a linear function exactly, so every ray's
integral is density_factor * chord * v(chord midpoint) (the chord and ray from
tests/pin_math.py, in fp64).  The adjoint of one ray's upstream gradient
spreads weights that sum to one per sample, so the gradient volume sums to
grad_out * density_factor * chord.  Tolerance 1e-4 relative, as for the
forward (fp32 storage of the affine values rounds them at ~1e-7).
"""
import numpy as np
import pytest

from cone_beam_ct_b200 import drr
from cone_beam_ct_b200 import workloads as wl
from tests import pin_math as pm

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
COEF = (0.01, 2e-5, -1e-5, 3e-5)     # a, b, c, d of the affine volume


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _affine(torch, n):
    a, b, c, d = COEF
    i = torch.arange(n, device="cuda", dtype=torch.float32)
    return (a + b * i[None, None, :] + c * i[None, :, None] + d * i[:, None, None]).contiguous()


def _geometry(n):
    sp = np.array([0.5, 0.5, 0.5], np.float32)
    origin = wl.centred_origin((n, n, n), sp).astype(np.float32)
    R = wl.random_rotation(np.random.default_rng(n))
    Rt = np.zeros((1, 3, 4))
    Rt[0, :, :3] = R
    Rt[0, :, 3] = [3.0, -2.0, 3.0 * n * 0.5]
    U, _, Vt = np.linalg.svd(Rt[0, :, :3])
    Rt[0, :, :3] = U @ Vt
    H = W = 24
    f = 0.7 * H * 3.0 / 1.0
    K = wl.intrinsics(f, f, (W - 1) / 2.0, (H - 1) / 2.0)
    return sp, origin, K, Rt, H, W


def _expected(n, sp, origin, K, Rt, H, W, df):
    lo = origin.astype(np.float64)
    hi = lo + (n - 1) * sp.astype(np.float64)
    a, b, c, d = COEF
    img = np.zeros((H, W))
    chords = np.zeros((H, W))
    for r in range(H):
        for cc in range(W):
            C, dd = pm.world_ray(K, Rt[0].reshape(-1), cc, r)
            ch = pm.box_chord(C, dd, lo, hi)
            if ch is None:
                continue
            mid = (C + 0.5 * (ch[0] + ch[1]) * dd - lo) / sp
            img[r, cc] = df * (ch[1] - ch[0]) * (a + b * mid[0] + c * mid[1] + d * mid[2])
            chords[r, cc] = ch[1] - ch[0]
    return img, chords


@pytest.mark.parametrize("layout,dtype,n", [(drr.DRR_LAYOUT_LINEAR, drr.DRR_F32, 1290),
                                            (drr.DRR_LAYOUT_PADDED, drr.DRR_F32, 1288),
                                            (drr.DRR_LAYOUT_CORNERS, drr.DRR_BF16, 646)])
def test_forward_at_the_largest_volume(cuda, layout, dtype, n):
    torch = cuda
    assert drr.drr_prepared_bytes((n, n, n), dtype, layout) > 0
    assert drr.drr_prepared_bytes((n + 1, n + 1, n + 1), dtype, layout) == 0   # one more is refused
    sp, origin, K, Rt, H, W = _geometry(n)
    vol = _affine(torch, n)
    if layout == drr.DRR_LAYOUT_LINEAR and dtype == drr.DRR_F32:
        src = vol
    else:
        src = torch.empty(drr.drr_prepared_bytes((n, n, n), dtype, layout), dtype=torch.uint8,
                          device="cuda")
        drr.drr_prepare_volume(vol, (n, n, n), dtype, layout, src)
    del vol
    Rt_d = torch.from_numpy(Rt.reshape(1, 12).astype(np.float32)).cuda()
    out = torch.empty((1, H, W), device="cuda")
    df = 1.0
    drr.drr_render(src, dtype, layout, (n, n, n), sp, origin, K, Rt_d, 1, H, W, 512, df,
                   wl.MODE_RAW, out)
    torch.cuda.synchronize()
    img, chords = _expected(n, sp, origin, K, Rt_d.cpu().numpy().astype(np.float64).reshape(1, 3, 4),
                            H, W, df)
    got = out.cpu().numpy()[0].astype(np.float64)
    assert np.count_nonzero(chords) > H * W // 2
    # bf16 storage rounds the affine values: its tolerance is the bf16 one
    tol = 1e-4 if dtype == drr.DRR_F32 else 1e-2
    assert np.max(np.abs(got - img)) <= tol * np.max(np.abs(img))
    del src
    torch.cuda.empty_cache()


def test_adjoint_at_the_largest_volume(cuda):
    torch = cuda
    n = 1290
    sp, origin, K, Rt, H, W = _geometry(n)
    Rt_d = torch.from_numpy(Rt.reshape(1, 12).astype(np.float32)).cuda()
    _, chords = _expected(n, sp, origin, K, Rt_d.cpu().numpy().astype(np.float64).reshape(1, 3, 4),
                          H, W, 1.0)
    r, c = np.unravel_index(np.argmax(chords), chords.shape)
    go = torch.zeros((1, H, W), device="cuda")
    go[0, r, c] = 0.75
    grad = torch.zeros((n, n, n), device="cuda")
    # the direct path (the workspace path's records would take 68 GB here)
    drr.drr_render_adjoint((n, n, n), sp, origin, K, Rt_d, 1, H, W, 512, 1.0, wl.MODE_RAW, go,
                           None, grad)
    torch.cuda.synchronize()
    total = grad.double().sum().item()
    assert abs(total - 0.75 * chords[r, c]) <= 1e-4 * 0.75 * chords[r, c]
    del grad
    torch.cuda.empty_cache()

"""GPU forward parity: the CUDA path (through the C ABI) against the fp64
oracle on the same seeded inputs.

Tolerance (the stated bar: max relative error 1e-4 on the integral for fp32
volumes, 1e-2 for bf16 volumes), read as two checks on every image:
normwise max |gpu - oracle| / max |oracle| <= tol, and per-pixel relative
error <= tol on pixels with |oracle| >= 1e-2 max |oracle|.  Beer-Lambert
images are compared directly: d(1 - e^-I)/dI = e^-I <= 1 and
(1 - e^-I) >= I e^-I, so their relative error never exceeds that of I.
bf16 volumes are checked twice: against the oracle fed the same
bf16-rounded values (kernel error alone, tol 1e-4) and against the oracle
fed the original fp32 values (storage + kernel error, tol 1e-2).
"""
import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import (BF16, BRICKS, CORNERS, F32, LAYOUTS, LINEAR, PADDED, QUADS, assert_parity,
                               bf16_values, gpu_forward, gpu_forward_staged)

pytestmark = pytest.mark.gpu
TOL_F32, TOL_BF16 = 1e-4, 1e-2


def _oracle(w, mode=None, vol=None, Rt=None):
    return oracle.render(w.vol if vol is None else vol, w.dims, w.spacing, w.origin, w.K,
                         w.Rt if Rt is None else Rt, w.H, w.W, w.n_samples, w.density_factor,
                         w.mode if mode is None else mode)


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from cone_beam_ct_b200 import drr
    drr.lib()
    return torch


CASES = [dict(seed=101), dict(seed=102, dims=(40, 9, 31), H=33, W=71, n_samples=50),
         dict(seed=103, dims=(2, 3, 2), H=17, W=16, n_samples=3),
         dict(seed=104, dims=(64, 48, 20), B=5, H=48, W=40, n_samples=1)]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
def test_small_ragged_fp32(cuda, case, layout, mode):
    w = wl.small_random_case(**CASES[case])
    got = gpu_forward(w, layout=layout, dtype=F32, mode=mode)
    ref = _oracle(w, mode=mode)
    assert np.count_nonzero(ref) > 0.05 * ref.size
    assert_parity(got, ref, TOL_F32, what=f"case {case}")
    # misses are exact zeros on both sides
    assert np.all(got[ref == 0.0] == 0.0)


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("layout", LAYOUTS)
def test_small_ragged_bf16(cuda, case, layout):
    w = wl.small_random_case(**CASES[case])
    got = gpu_forward(w, layout=layout, dtype=BF16, mode=wl.MODE_RAW)
    assert_parity(got, _oracle(w, mode=wl.MODE_RAW, vol=bf16_values(w.vol)), TOL_F32,
                  what="vs oracle on bf16 values")
    assert_parity(got, _oracle(w, mode=wl.MODE_RAW), TOL_BF16, what="vs oracle on fp32 values")


@pytest.mark.parametrize("layout", LAYOUTS)
def test_config1_full_image(cuda, layout):
    w = wl.make_config(1)
    got = gpu_forward(w, layout=layout)
    assert_parity(got, _oracle(w), TOL_F32, what="config 1")


_CFG2 = {}


def _config2_oracle(mode):
    if mode not in _CFG2:
        w = wl.make_config(2)
        _CFG2[mode] = (w, _oracle(w, mode=mode))
    return _CFG2[mode]


@pytest.mark.slow
@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("mode", [wl.MODE_BEER_LAMBERT, wl.MODE_RAW])
def test_config2_full_image(cuda, layout, mode):
    w, ref = _config2_oracle(mode)
    assert_parity(gpu_forward(w, layout=layout, mode=mode), ref, TOL_F32,
                  what=f"config 2 layout {layout} mode {mode}")


def _sampled_ids(w, n, seed):
    """Random rays plus every view's four image corners, edge midpoints and centre."""
    rng = np.random.default_rng(seed)
    ids = set(rng.choice(w.rays, size=n, replace=False).tolist())
    for b in range(w.B):
        for r in (0, w.H // 2, w.H - 1):
            for c in (0, w.W // 2, w.W - 1):
                ids.add((b * w.H + r) * w.W + c)
    return np.array(sorted(ids), dtype=np.int64)


def _sampled_oracle(w, ids, vol=None, mode=None):
    return oracle.render_rays(w.vol if vol is None else vol, w.dims, w.spacing, w.origin, w.K,
                              w.Rt, w.H, w.W, w.n_samples, w.density_factor,
                              w.mode if mode is None else mode, ids)


@pytest.mark.slow
@pytest.mark.parametrize("layout", [PADDED, CORNERS, BRICKS])
def test_config3_bf16_sampled(cuda, layout):
    w = wl.make_config(3)
    got = gpu_forward(w, layout=layout, dtype=BF16).reshape(-1)
    ids = _sampled_ids(w, 40000, 3)
    assert_parity(got[ids], _sampled_oracle(w, ids, vol=bf16_values(w.vol)), TOL_F32,
                  what="config 3 vs oracle on bf16 values")
    assert_parity(got[ids], _sampled_oracle(w, ids), TOL_BF16, what="config 3 vs fp32 values")
    # property at full size: Beer-Lambert images lie in [0, 1)
    assert np.all(got >= 0.0) and np.all(got < 1.0)


@pytest.mark.slow
def test_config4_hbm_sampled(cuda):
    w = wl.make_config(4)
    ids = _sampled_ids(w, 30000, 4)
    ref = _sampled_oracle(w, ids)
    for layout in LAYOUTS:
        got = gpu_forward(w, layout=layout).reshape(-1)
        assert_parity(got[ids], ref, TOL_F32, what=f"config 4 layout {layout}")


def test_layouts_agree(cuda):
    w = wl.small_random_case(105, H=64, W=64)
    for dtype in (F32, BF16):
        a = gpu_forward(w, layout=LINEAR, dtype=dtype)
        # same positions, fractions and lerps: corner records and quads are bit-identical
        assert np.array_equal(a, gpu_forward(w, layout=CORNERS, dtype=dtype))
        assert np.array_equal(a, gpu_forward(w, layout=QUADS, dtype=dtype))
        assert np.array_equal(a, gpu_forward(w, layout=BRICKS, dtype=dtype))
        assert_parity(a, gpu_forward(w, layout=PADDED, dtype=dtype), 1e-5, what="linear vs padded")


def _inside_camera(w):
    """The same case with the camera moved inside the volume (near its centre)."""
    Rt = w.Rt.astype(np.float64).reshape(-1, 3, 4).copy()
    centre = np.asarray(w.origin, np.float64) + 0.5 * (np.asarray(w.dims) - 1) * np.asarray(
        w.spacing, np.float64) + np.array([0.31, -0.17, 0.23])
    for b in range(Rt.shape[0]):
        Rt[b, :, 3] = -Rt[b, :, :3] @ centre
    w.Rt = Rt.astype(np.float32)
    return w


# geometries for the bricked forward, whose integral modes stage each layer
# of a tile's bricks in shared memory: ragged small volumes, rays a voxel
# apart and rays much closer (staged layers), a wide-angle camera (layers
# wider than the staging window: global reads), a camera inside the volume
STAGED_CASES = {
    "small ragged": lambda: wl.small_random_case(131),
    "sparse rays, 40 views": lambda: wl.small_random_case(132, dims=(70, 66, 75), B=40, H=48,
                                                          W=40, n_samples=90),
    "dense rays": lambda: wl.small_random_case(133, dims=(23, 17, 29), H=150, W=170,
                                               n_samples=40),
    "wide angle": lambda: _wide_angle(wl.small_random_case(134, dims=(90, 80, 70), H=64, W=64)),
    "camera inside": lambda: _inside_camera(wl.small_random_case(135, dims=(40, 44, 36))),
}


def _wide_angle(w):
    K = np.asarray(w.K, np.float32).reshape(3, 3).copy()
    K[0, 0] /= 8.0
    K[1, 1] /= 8.0
    w.K = K.reshape(-1)
    return w


@pytest.mark.parametrize("name", sorted(STAGED_CASES))
@pytest.mark.parametrize("mode", [wl.MODE_RAW, wl.MODE_BEER_LAMBERT])
def test_staged_bricks_match_the_linear_layout_bit_for_bit(cuda, name, mode):
    # staged and global samples read the same 8 voxels and take the same lerps
    w = STAGED_CASES[name]()
    for dtype in (F32, BF16):
        a = gpu_forward(w, layout=LINEAR, dtype=dtype, mode=mode)
        got = gpu_forward(w, layout=BRICKS, dtype=dtype, mode=mode)
        assert np.array_equal(a, got), f"{name}: {np.count_nonzero(a != got)} pixels differ"
        staged = gpu_forward_staged(w, dtype=dtype, mode=mode)
        assert np.array_equal(a, staged), f"{name}: {np.count_nonzero(a != staged)} pixels differ"
    ref = oracle.render(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                        w.density_factor, mode)
    assert_parity(gpu_forward(w, layout=BRICKS, dtype=F32, mode=mode), ref, TOL_F32, what=name)


def test_forward_is_deterministic(cuda):
    w = wl.small_random_case(106)
    assert np.array_equal(gpu_forward(w), gpu_forward(w))


def test_camera_inside_volume_and_axis_parallel_rays(cuda):
    # camera at the volume centre looking along +z: principal ray parallel to two axes,
    # half the image rays start inside the box (t0 = 0)
    w = wl.small_random_case(107, dims=(24, 20, 28), H=21, W=19)
    Rt = np.zeros((2, 3, 4), np.float32)
    Rt[0, :, :3] = np.eye(3)
    Rt[1, :, :3] = np.array([[0, 1, 0], [0, 0, 1], [1, 0, 0]])   # looks along world +x
    Rt[1, :, 3] = [0.0, 0.0, 30.0]
    K = wl.intrinsics(12.0, 12.0, 9.0, 10.0)
    w.K, w.Rt = K, Rt
    for layout in LAYOUTS:
        got = gpu_forward(w, layout=layout, mode=wl.MODE_RAW)
        assert_parity(got, _oracle(w, mode=wl.MODE_RAW), TOL_F32, what="inside/axis")


def test_non_finite_pose_gives_zero_image(cuda):
    w = wl.small_random_case(108)
    Rt = w.Rt.copy()
    Rt[1, 0, 0] = np.nan
    Rt[2, 2, 3] = np.inf
    for layout in LAYOUTS:
        got = gpu_forward(w, layout=layout, Rt=Rt)
        assert np.all(got[1] == 0.0) and np.all(got[2] == 0.0)
        assert_parity(got[0], _oracle(w, Rt=w.Rt[:1])[0], TOL_F32)


def test_empty_batch_writes_nothing(cuda):
    import torch
    from cone_beam_ct_b200 import drr
    w = wl.small_random_case(109)
    v, Rt = torch.zeros(4, device="cuda"), torch.zeros(12, device="cuda")
    out = torch.full((4,), 7.0, device="cuda")
    drr.drr_render(v, F32, LINEAR, w.dims, w.spacing, w.origin, w.K, Rt, 0, w.H, w.W,
                   w.n_samples, 1.0, 0, out)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_runs_on_a_side_stream(cuda):
    import torch
    w = wl.small_random_case(110)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        got = gpu_forward(w)
    assert_parity(got, _oracle(w), TOL_F32)


def test_prepare_layouts_round_trip(cuda):
    import torch
    from cone_beam_ct_b200 import drr
    w = wl.small_random_case(111, dims=(7, 5, 6))
    v = torch.from_numpy(w.vol).cuda()
    nx, ny, nz = w.dims
    for dtype, np_t, conv in ((F32, np.float32, lambda a: a),
                              (BF16, np.uint16, lambda a: oracle.bf16_to_float(a))):
        expect = w.vol if dtype == F32 else bf16_values(w.vol)
        for layout in LAYOUTS:
            nbytes = drr.drr_prepared_bytes(w.dims, dtype, layout)
            buf = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device="cuda")
            drr.drr_prepare_volume(v, w.dims, dtype, layout, buf)
            torch.cuda.synchronize()
            a = conv(buf.cpu().numpy().view(np_t))
            if layout == LINEAR:
                assert np.array_equal(a.reshape(nz, ny, nx), expect)
            elif layout == PADDED:
                p = a.reshape(nz + 2, ny + 2, nx + 2)
                assert np.array_equal(p[1:-1, 1:-1, 1:-1], expect)
                border = p.copy()
                border[1:-1, 1:-1, 1:-1] = 0
                assert np.all(border == 0)
            elif layout == BRICKS:
                # voxel (8bx + lx, 8by + ly, 8bz + lz) of brick (bx, by, bz) at element
                # (lz * 9 + ly) * 9 + lx of a 736-element block, zero elsewhere
                nb = [-(-(n - 1) // 8) for n in (nx, ny, nz)]
                blocks = a.reshape(nb[2], nb[1], nb[0], 736)
                assert np.all(blocks[..., 729:] == 0)
                cube = blocks[..., :729].reshape(nb[2], nb[1], nb[0], 9, 9, 9)
                full = np.zeros((8 * nb[2] + 1, 8 * nb[1] + 1, 8 * nb[0] + 1), a.dtype)
                full[:nz, :ny, :nx] = expect
                for bz in range(nb[2]):
                    for by in range(nb[1]):
                        for bx in range(nb[0]):
                            assert np.array_equal(cube[bz, by, bx],
                                                  full[8 * bz:8 * bz + 9, 8 * by:8 * by + 9,
                                                       8 * bx:8 * bx + 9])
            elif layout == QUADS:
                # voxel (i + a, j + b, k) of quad (i, j, k) at element a + 2b
                rec = a.reshape(nz, ny - 1, nx - 1, 4)
                for e in range(4):
                    da, db = e & 1, e >> 1
                    assert np.array_equal(rec[..., e], expect[:, db:ny - 1 + db, da:nx - 1 + da])
            else:
                # corner (a, b, c) of cell (i, j, k) at element a + 2b + 4c
                rec = a.reshape(nz - 1, ny - 1, nx - 1, 8)
                for e in range(8):
                    da, db, dc = e & 1, (e >> 1) & 1, e >> 2
                    assert np.array_equal(rec[..., e],
                                          expect[dc:nz - 1 + dc, db:ny - 1 + db, da:nx - 1 + da])

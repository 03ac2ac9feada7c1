"""Seeded synthetic workloads for the cone-beam DRR ray-march.

This module only *makes inputs*: attenuation volumes (ellipsoid phantoms),
pinhole intrinsics K and world->camera extrinsics [R|t], and upstream image
gradients.  It holds none of the ray-march arithmetic, so both the CUDA path
and the fp64 CPU oracle can consume the very same arrays.

Everything is generated from ``numpy.random.default_rng(seed)`` with
seed = 1000 + config number, and every array handed out is float32: those
are the values the GPU sees, and the oracle widens exactly these values to
fp64.

Conventions (shared by both sides and stated once here):

* volume ``vol[k][j][i]`` (i fastest), dims ``(nx, ny, nz)``; world position
  of voxel (i, j, k) is ``origin + spacing * (i, j, k)`` (origin = centre of
  voxel 0).  "Centred" means ``origin = -(n - 1) / 2 * spacing``.
* pinhole camera in the Hartley-Zisserman form ``x ~ K [R | t] X`` (nanodrr
  page, introduction: all projective geometry uses the HZ pinhole); R, t map
  world to camera, camera +z looks into the scene, +y points down the image.
  Pixel (row r, column c) has its centre at (u, v) = (c, r).
* C-arm poses follow the flashdrr.rendering API docs, carm_to_camera_params
  (AP view: source anterior looking posterior; positive lateral angle = RAO,
  source to the patient's right; positive AP angle = caudal) in RAS world
  coordinates, with the volume centre at the world origin.
* HU -> mu follows the flashdrr transfer-function idea (flashdrr.rendering
  API docs, piecewise_linear_channelwise): a single linear segment
  mu = 0.02 * (1 + HU / 1000) per mm, clamped at 0.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

MODE_RAW = 0
MODE_BEER_LAMBERT = 1
MODE_ALPHA = 2

DTYPE_F32 = 0
DTYPE_BF16 = 1


# ---------------------------------------------------------------------------
# small geometry helpers (input construction only)
# ---------------------------------------------------------------------------

def rot_x(a: float) -> np.ndarray:
    c, s = math.cos(a), math.sin(a)
    return np.array([[1, 0, 0], [0, c, -s], [0, s, c]], dtype=np.float64)


def rot_y(a: float) -> np.ndarray:
    c, s = math.cos(a), math.sin(a)
    return np.array([[c, 0, s], [0, 1, 0], [-s, 0, c]], dtype=np.float64)


def rot_z(a: float) -> np.ndarray:
    c, s = math.cos(a), math.sin(a)
    return np.array([[c, -s, 0], [s, c, 0], [0, 0, 1]], dtype=np.float64)


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    """Uniformly distributed rotation from a normalised Gaussian quaternion."""
    q = rng.normal(size=4)
    q /= np.linalg.norm(q)
    w, x, y, z = q
    return np.array([
        [1 - 2 * (y * y + z * z), 2 * (x * y - z * w), 2 * (x * z + y * w)],
        [2 * (x * y + z * w), 1 - 2 * (x * x + z * z), 2 * (y * z - x * w)],
        [2 * (x * z - y * w), 2 * (y * z + x * w), 1 - 2 * (x * x + y * y)],
    ])


def intrinsics(fx: float, fy: float, cx: float, cy: float, skew: float = 0.0) -> np.ndarray:
    """Upper-triangular HZ intrinsics, row-major 3x3, float32."""
    return np.array([[fx, skew, cx], [0.0, fy, cy], [0.0, 0.0, 1.0]], dtype=np.float32)


def look_at_extrinsics(cam_pos: Sequence[float], focal: Sequence[float],
                       up: Sequence[float]) -> np.ndarray:
    """World->camera [R|t] (3x4, float64) for a camera at ``cam_pos`` looking at
    ``focal``.  Camera axes: z = forward, y = -(up made orthogonal to z),
    x = y cross z (right-handed, image rows grow downwards)."""
    cam_pos = np.asarray(cam_pos, dtype=np.float64)
    fwd = np.asarray(focal, dtype=np.float64) - cam_pos
    fwd /= np.linalg.norm(fwd)
    up = np.asarray(up, dtype=np.float64)
    up_perp = up - np.dot(up, fwd) * fwd
    up_perp /= np.linalg.norm(up_perp)
    y_axis = -up_perp
    x_axis = np.cross(y_axis, fwd)
    R = np.stack([x_axis, y_axis, fwd], axis=0)
    t = -R @ cam_pos
    return np.concatenate([R, t[:, None]], axis=1)


def carm_camera(lat_deg: float, ap_deg: float, source_to_centre: float,
                centre: Sequence[float] = (0.0, 0.0, 0.0),
                table_si: float = 0.0) -> np.ndarray:
    """[R|t] for a C-arm source ``source_to_centre`` mm from the volume centre.

    RAS world: +x right, +y anterior, +z superior.  lat = 0, ap = 0 puts the
    source anterior, looking posterior, with superior as image "up".
    Positive lat moves the source to the patient's right (RAO); positive ap
    tilts it inferiorly (caudal).  A table shift moves the patient (and so
    the look-at point) along the superior axis.
    """
    th, ph = math.radians(lat_deg), math.radians(ap_deg)
    c = np.asarray(centre, dtype=np.float64) + np.array([0.0, 0.0, table_si])
    direction = np.array([math.cos(ph) * math.sin(th),
                          math.cos(ph) * math.cos(th),
                          -math.sin(ph)])
    pos = c + source_to_centre * direction
    return look_at_extrinsics(pos, c, (0.0, 0.0, 1.0))


def centred_origin(dims: Sequence[int], spacing: Sequence[float]) -> np.ndarray:
    return np.array([-(n - 1) / 2.0 * s for n, s in zip(dims, spacing)], dtype=np.float32)


# ---------------------------------------------------------------------------
# phantoms
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Ellipsoid:
    centre: np.ndarray      # world mm
    semi_axes: np.ndarray   # mm, along the ellipsoid's own axes
    rotation: np.ndarray    # columns = ellipsoid axes in world
    value: float            # additive value (HU or mu)


def _index_range(centre, half, origin, spacing, n):
    lo = int(np.floor((centre - half - origin) / spacing)) - 1
    hi = int(np.ceil((centre + half - origin) / spacing)) + 2
    return max(lo, 0), min(hi, n)


def _inside_box(e: Ellipsoid, spacing, origin, rng) -> np.ndarray:
    """Voxel centres of the index box ``rng`` that lie inside ``e``.  The
    ellipsoid-frame coordinates are sums of per-axis terms, so the quadratic
    form is assembled from 1-D coordinate vectors by broadcasting."""
    axes = [origin[a] + spacing[a] * np.arange(rng[a][0], rng[a][1], dtype=np.float64)
            - e.centre[a] for a in range(3)]
    X = axes[0][None, None, :]
    Y = axes[1][None, :, None]
    Z = axes[2][:, None, None]
    q = np.zeros((len(axes[2]), len(axes[1]), len(axes[0])))
    for m in range(3):      # coordinate along the ellipsoid's m-th axis
        loc = X * e.rotation[0, m] + Y * e.rotation[1, m] + Z * e.rotation[2, m]
        q += (loc / e.semi_axes[m]) ** 2
    return q <= 1.0


def _add_ellipsoid(out: np.ndarray, dims, spacing, origin, e: Ellipsoid,
                   mask: Optional[Ellipsoid] = None) -> None:
    """out[k][j][i] += e.value where the voxel centre lies inside e (and
    inside ``mask``), evaluated on the ellipsoid's bounding box only."""
    half = np.sqrt(((e.rotation * e.semi_axes[None, :]) ** 2).sum(axis=1))
    rng = [_index_range(e.centre[a], half[a], origin[a], spacing[a], dims[a]) for a in range(3)]
    if any(lo >= hi for lo, hi in rng):
        return
    inside = _inside_box(e, spacing, origin, rng)
    if mask is not None:
        inside &= _inside_box(mask, spacing, origin, rng)
    out[rng[2][0]:rng[2][1], rng[1][0]:rng[1][1], rng[0][0]:rng[0][1]] += inside * e.value


def voxelize(dims: Sequence[int], spacing: Sequence[float], origin: Sequence[float],
             ellipsoids: Sequence[Ellipsoid], background: float = 0.0,
             mask: Optional[Ellipsoid] = None) -> np.ndarray:
    """Sum of ellipsoid indicator functions (voxel centre inside) times value,
    on a ``vol[k][j][i]`` float64 grid.  ``mask`` (optional) zeroes the
    ellipsoid contributions outside another ellipsoid."""
    nx, ny, nz = (int(n) for n in dims)
    sp = np.asarray(spacing, dtype=np.float64)
    org = np.asarray(origin, dtype=np.float64)
    out = np.full((nz, ny, nx), background, dtype=np.float64)
    for e in ellipsoids:
        _add_ellipsoid(out, (nx, ny, nz), sp, org, e, mask)
    return out


def hu_to_mu(hu: np.ndarray) -> np.ndarray:
    """mu per mm = 0.02 * (1 + HU / 1000), clamped at 0 (water 0.02/mm)."""
    return np.maximum(0.0, 0.02 * (1.0 + hu / 1000.0))


def shepp_logan_style_ellipsoids(rng: np.random.Generator, half_extent_mm: float = 128.0
                                 ) -> List[Ellipsoid]:
    """10 ellipsoids in HU for a cube of side 2*half_extent_mm: a dense outer
    shell (+2000 HU over a -1000 HU background), an inner body (-1000 HU,
    0.9x the outer), and 8 interior features (semi-axes 8..48 mm, random
    orientation, centres inside the inner body, dHU in [-200, +1000]).
    A seeded *style* of a head phantom, not a published phantom table."""
    outer_axes = rng.uniform(0.80, 0.95, size=3) * half_extent_mm
    eye = np.eye(3)
    ells = [Ellipsoid(np.zeros(3), outer_axes, eye, 2000.0),
            Ellipsoid(np.zeros(3), 0.9 * outer_axes, eye, -1000.0)]
    inner_axes = 0.9 * outer_axes
    for _ in range(8):
        while True:                                # centre inside the inner body
            c = rng.uniform(-1.0, 1.0, size=3)
            if np.sum(c * c) <= 1.0:
                break
        centre = c * inner_axes
        axes = rng.uniform(8.0, 48.0, size=3)
        rot = random_rotation(rng)
        dhu = rng.uniform(-200.0, 1000.0)
        ells.append(Ellipsoid(centre, axes, rot, dhu))
    return ells


def shepp_logan_style_mu(n: int, spacing_mm: float, rng: np.random.Generator,
                         noise_frac: float = 0.0) -> np.ndarray:
    """mu volume (float32, [nz][ny][nx]) of the HU phantom on an n^3 grid."""
    dims = (n, n, n)
    sp = (spacing_mm,) * 3
    origin = centred_origin(dims, sp).astype(np.float64)
    ells = shepp_logan_style_ellipsoids(rng)
    hu = voxelize(dims, sp, origin, ells, background=-1000.0)
    np.clip(hu, -1000.0, 2000.0, out=hu)
    mu = hu_to_mu(hu).astype(np.float32)
    if noise_frac > 0.0:
        for k in range(n):                          # multiplicative: air stays 0
            mu[k] *= (1.0 + rng.uniform(-noise_frac, noise_frac, size=(n, n))).astype(np.float32)
    return mu


def sphere_ellipsoid_mu(rng: np.random.Generator) -> np.ndarray:
    """64^3, 2 mm: a 28-voxel-radius sphere of mu 0.02/mm plus 6 random
    ellipsoids (semi-axes 5..25 voxels, additive mu 0.005..0.03/mm, centres in
    a 14-voxel ball) masked by the sphere."""
    n, sp = 64, 2.0
    dims, spacing = (n, n, n), (sp, sp, sp)
    origin = centred_origin(dims, spacing).astype(np.float64)
    sphere = Ellipsoid(np.zeros(3), np.full(3, 28.0 * sp), np.eye(3), 0.02)
    ells = []
    for _ in range(6):
        while True:
            c = rng.uniform(-1.0, 1.0, size=3)
            if np.sum(c * c) <= 1.0:
                break
        ells.append(Ellipsoid(c * 14.0 * sp, rng.uniform(5.0, 25.0, size=3) * sp,
                              random_rotation(rng), rng.uniform(0.005, 0.03)))
    base = voxelize(dims, spacing, origin, [sphere])
    extra = voxelize(dims, spacing, origin, ells, mask=sphere)
    return (base + extra).astype(np.float32)


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    vol: np.ndarray            # float32 [nz][ny][nx]
    dims: Tuple[int, int, int]
    spacing: np.ndarray        # float32 (3,)
    origin: np.ndarray         # float32 (3,)
    K: np.ndarray              # float32 (3,3)
    Rt: np.ndarray             # float32 (B,3,4)
    H: int
    W: int
    n_samples: int
    density_factor: float
    mode: int
    dtype: int                 # storage dtype of the volume on the GPU
    grad_out: Optional[np.ndarray] = None   # float32 (B,H,W) upstream gradient

    @property
    def B(self) -> int:
        return int(self.Rt.shape[0])

    @property
    def rays(self) -> int:
        return self.B * self.H * self.W

    @property
    def samples(self) -> int:
        return self.rays * self.n_samples


SOURCE_TO_ISO_MM = 510.0
SDD_MM = 1020.0


def _euler_views(rng, n_views, max_deg=30.0, max_shift=20.0):
    Rt = np.empty((n_views, 3, 4), dtype=np.float64)
    for v in range(n_views):
        a, b, g = np.radians(rng.uniform(-max_deg, max_deg, size=3))
        R = rot_z(g) @ rot_y(b) @ rot_x(a)
        t = rng.uniform(-max_shift, max_shift, size=3) + np.array([0.0, 0.0, SOURCE_TO_ISO_MM])
        Rt[v, :, :3] = R
        Rt[v, :, 3] = t
    return Rt.astype(np.float32)


def _carm_views(rng, n_views):
    Rt = np.empty((n_views, 3, 4), dtype=np.float64)
    for v in range(n_views):
        lat = rng.uniform(-90.0, 90.0)
        ap = rng.uniform(-45.0, 45.0)
        Rt[v] = carm_camera(lat, ap, SOURCE_TO_ISO_MM)
    return Rt.astype(np.float32)


def _detector_K(n_px: int, pixel_mm: float) -> np.ndarray:
    f = SDD_MM / pixel_mm
    c = (n_px - 1) / 2.0
    return intrinsics(f, f, c, c)


CONFIG_NAMES = {
    1: "64^3 fp32 sphere+ellipsoids, 1 view 64x64, 64 samples, Beer-Lambert",
    2: "256^3 fp32 HU phantom, 64 views 200x200, 256 samples, Beer-Lambert",
    3: "256^3 bf16 HU phantom, 4 C-arm views 1024x1024, 512 samples, Beer-Lambert",
    4: "512^3 fp32 HU phantom +-2% noise, 2 C-arm views 2048x2048, 256 samples, raw",
    5: "adjoint of 256^3 / 64 views 200x200 / 256 samples, raw, N(0,1) upstream",
}


def make_config(index: int, seed: Optional[int] = None) -> Workload:
    """The five seeded workloads (seed defaults to 1000 + index)."""
    rng = np.random.default_rng(1000 + index if seed is None else seed)
    if index == 1:
        vol = sphere_ellipsoid_mu(rng)
        dims, sp = (64, 64, 64), np.full(3, 2.0, dtype=np.float32)
        Rt = np.zeros((1, 3, 4), dtype=np.float32)
        Rt[0, :, :3] = np.eye(3)
        Rt[0, :, 3] = (0.0, 0.0, SOURCE_TO_ISO_MM)
        return Workload(CONFIG_NAMES[1], vol, dims, sp, centred_origin(dims, sp),
                        _detector_K(64, 4.0), Rt, 64, 64, 64, 1.0, MODE_BEER_LAMBERT, DTYPE_F32)
    if index in (2, 5):
        vol = shepp_logan_style_mu(256, 1.0, rng)
        dims, sp = (256, 256, 256), np.full(3, 1.0, dtype=np.float32)
        Rt = _euler_views(rng, 64)
        mode = MODE_BEER_LAMBERT if index == 2 else MODE_RAW
        w = Workload(CONFIG_NAMES[index], vol, dims, sp, centred_origin(dims, sp),
                     _detector_K(200, 2.0), Rt, 200, 200, 256, 1.0, mode, DTYPE_F32)
        if index == 5:
            w.grad_out = rng.standard_normal(size=(64, 200, 200)).astype(np.float32)
        return w
    if index == 3:
        vol = shepp_logan_style_mu(256, 1.0, rng)
        dims, sp = (256, 256, 256), np.full(3, 1.0, dtype=np.float32)
        Rt = _carm_views(rng, 4)
        return Workload(CONFIG_NAMES[3], vol, dims, sp, centred_origin(dims, sp),
                        _detector_K(1024, 0.4), Rt, 1024, 1024, 512, 1.0,
                        MODE_BEER_LAMBERT, DTYPE_BF16)
    if index == 4:
        vol = shepp_logan_style_mu(512, 0.5, rng, noise_frac=0.02)
        dims, sp = (512, 512, 512), np.full(3, 0.5, dtype=np.float32)
        Rt = _carm_views(rng, 2)
        return Workload(CONFIG_NAMES[4], vol, dims, sp, centred_origin(dims, sp),
                        _detector_K(2048, 0.2), Rt, 2048, 2048, 256, 1.0, MODE_RAW, DTYPE_F32)
    raise ValueError(f"unknown config {index}")


def small_random_case(seed: int, dims=(23, 17, 29), B=3, H=37, W=45, n_samples=33,
                      spacing=(1.1, 0.9, 1.3), mode=MODE_BEER_LAMBERT,
                      dtype=DTYPE_F32) -> Workload:
    """A small, deliberately ragged case (odd sizes, anisotropic voxels,
    random poses around the volume) that still spans several pixel tiles and
    leaves ragged tile tails.  Values are U(0, 0.05) per mm."""
    rng = np.random.default_rng(seed)
    nx, ny, nz = dims
    vol = rng.uniform(0.0, 0.05, size=(nz, ny, nx)).astype(np.float32)
    sp = np.asarray(spacing, dtype=np.float32)
    origin = (centred_origin(dims, sp) + rng.uniform(-2, 2, size=3)).astype(np.float32)
    extent = float(np.max(np.asarray(dims) * sp))
    dist = 3.0 * extent
    Rt = np.empty((B, 3, 4), dtype=np.float64)
    for b in range(B):
        R = random_rotation(rng)
        centre_cam = np.array([rng.uniform(-0.1, 0.1) * extent,
                               rng.uniform(-0.1, 0.1) * extent, dist])
        Rt[b, :, :3] = R
        Rt[b, :, 3] = centre_cam        # X_cam = R X + t: the world origin sits at centre_cam
    # focal length so that the volume fills ~80% of the image
    f = 0.8 * min(H, W) * dist / extent
    K = intrinsics(f, f * 1.05, (W - 1) / 2.0 + 0.3, (H - 1) / 2.0 - 0.2, skew=0.5)
    return Workload(f"random-{seed}", vol, tuple(dims), sp, origin, K, Rt.astype(np.float32),
                    H, W, n_samples, 0.7, mode, dtype)

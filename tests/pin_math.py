"""Independent test-side mathematics used to pin the oracle.

Nothing here calls the oracle or the CUDA path.  Each routine reaches its
answer by a different route from the oracle's: rays from a library linear
solve of the projection equation instead of back substitution, box chords by
enumerating face intersections instead of slab min/max, the exact integral
of the trilinear interpolant by splitting the ray at voxel planes and using
2-point Gauss-Legendre per piece instead of the midpoint sum.
"""
import numpy as np


def world_ray(K, Rt12, u, v):
    """Camera centre and unit direction (world) of pixel centre (u, v),
    solving (K R) d ~ (u, v, 1) and R C + t = 0 with numpy.linalg.solve."""
    K = np.asarray(K, dtype=np.float64).reshape(3, 3)
    Rt = np.asarray(Rt12, dtype=np.float64).reshape(3, 4)
    R, t = Rt[:, :3], Rt[:, 3]
    C = np.linalg.solve(R, -t)
    d = np.linalg.solve(K @ R, np.array([u, v, 1.0]))
    if np.dot(R @ d, [0, 0, 1]) < 0:           # in front of the camera: camera z > 0
        d = -d
    return C, d / np.linalg.norm(d)


def project(K, Rt12, X):
    """Pixel coordinates and depth of world point X under P = K [R | t]."""
    P = np.asarray(K, dtype=np.float64).reshape(3, 3) @ np.asarray(Rt12, np.float64).reshape(3, 4)
    x = P @ np.append(np.asarray(X, dtype=np.float64), 1.0)
    return x[0] / x[2], x[1] / x[2], x[2]


def box_chord(C, d, lo, hi):
    """Parameter interval [ta, tb] (t >= 0) of the line C + t d inside the
    axis-aligned box [lo, hi], found by intersecting the line with each of
    the six face rectangles.  Returns None when the ray does not cross the
    box with positive length."""
    C, d, lo, hi = (np.asarray(a, dtype=np.float64) for a in (C, d, lo, hi))
    ts = []
    tol = 1e-9 * (1.0 + np.max(np.abs(hi - lo)))
    for a in range(3):
        if d[a] == 0.0:
            continue
        for plane in (lo[a], hi[a]):
            t = (plane - C[a]) / d[a]
            X = C + t * d
            others = [b for b in range(3) if b != a]
            if all(lo[b] - tol <= X[b] <= hi[b] + tol for b in others):
                ts.append(t)
    inside_start = np.all(C >= lo) and np.all(C <= hi)
    if inside_start:
        ts.append(0.0)
    ts = [t for t in ts if t >= 0.0]
    if len(ts) < 2:
        return None
    ta, tb = min(ts), max(ts)
    if tb - ta <= 0.0:
        return None
    return ta, tb


def trilinear_zero_padded(vol, p):
    """Zero-padded trilinear interpolation of vol[k][j][i] at IJK point p."""
    nz, ny, nx = vol.shape
    i0 = np.floor(p).astype(np.int64)
    f = np.asarray(p, dtype=np.float64) - i0
    s = 0.0
    for dk in (0, 1):
        for dj in (0, 1):
            for di in (0, 1):
                i, j, k = i0[0] + di, i0[1] + dj, i0[2] + dk
                if 0 <= i < nx and 0 <= j < ny and 0 <= k < nz:
                    w = ((f[0] if di else 1 - f[0]) * (f[1] if dj else 1 - f[1])
                         * (f[2] if dk else 1 - f[2]))
                    s += w * float(vol[k, j, i])
    return s


def exact_line_integral(vol, P0, D, ta, tb):
    """Exact integral over t in [ta, tb] of trilinear(vol, P0 + t D).

    Between consecutive crossings of integer planes the integrand is a
    product of three linear factors (a cubic), which 2-point Gauss-Legendre
    integrates exactly."""
    P0 = np.asarray(P0, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    cuts = [ta, tb]
    for a in range(3):
        if D[a] == 0.0:
            continue
        pa, pb = P0[a] + ta * D[a], P0[a] + tb * D[a]
        lo, hi = min(pa, pb), max(pa, pb)
        for m in range(int(np.ceil(lo)), int(np.floor(hi)) + 1):
            t = (m - P0[a]) / D[a]
            if ta < t < tb:
                cuts.append(t)
    cuts = np.unique(np.array(cuts))
    g = 1.0 / np.sqrt(3.0)
    total = 0.0
    for a, b in zip(cuts[:-1], cuts[1:]):
        mid, half = 0.5 * (a + b), 0.5 * (b - a)
        for x in (-g, g):
            total += half * trilinear_zero_padded(vol, P0 + (mid + half * x) * D)
    return total

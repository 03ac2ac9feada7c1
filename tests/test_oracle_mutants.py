"""The oracle's pins must fail on plausible slips (CPU only).

Each case plants one mistake in a temporary copy of the oracle's C source,
builds it, and runs the pin suite against that copy in a subprocess
(DRR_ORACLE_LIB points the oracle binding at the mutant).  A mutant that
passes every pin would mean the pins leave that part of the oracle unchecked.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "drr_oracle.c")

MUTANTS = {
    "trilinear weights f <-> 1-f": (
        "(di ? f[0] : 1.0 - f[0]) * (dj ? f[1] : 1.0 - f[1]) *\n"
        "                           (dk ? f[2] : 1.0 - f[2]);\n                s += w",
        "(di ? 1.0 - f[0] : f[0]) * (dj ? f[1] : 1.0 - f[1]) *\n"
        "                           (dk ? f[2] : 1.0 - f[2]);\n                s += w"),
    "left-endpoint instead of midpoint samples": (
        "return t0 + ((double)i + 0.5) * dt;", "return t0 + ((double)i) * dt;"),
    "camera centre sign": ("C[a] = -ca;", "C[a] = ca;"),
    "direction not normalised": ("for (int a = 0; a < 3; ++a) d[a] *= inv;", "(void)inv;"),
    "R instead of R^T": ("da += Rt[4 * r + a] * q[r];", "da += Rt[4 * a + r] * q[r];"),
    "box [0, n] instead of [0, n-1]": (
        "double lo = 0.0 - pad, hi = (double)(g->n[a] - 1) + pad;",
        "double lo = 0.0 - pad, hi = (double)(g->n[a]) + pad;"),
    "Beer-Lambert as exp(-I)": (
        "return mode == ORACLE_BEER_LAMBERT ? -expm1(-I) : I;",
        "return mode == ORACLE_BEER_LAMBERT ? exp(-I) : I;"),
    "adjoint without dt": (
        "double scale = go * density_factor * dt;", "double scale = go * density_factor;"),
    "adjoint i/j transposed": (
        "grad[(kk * g->n[1] + jj) * g->n[0] + ii] += scale * w;",
        "grad[(kk * g->n[1] + ii) * g->n[0] + jj] += scale * w;"),
    "no clamp of t0 at the camera": ("*t0 = t_near > 0.0 ? t_near : 0.0;", "*t0 = t_near;"),
    "half-pixel shift": (
        "double u = (double)(rc % job->W), v = (double)(rc / job->W);",
        "double u = (double)(rc % job->W) + 0.5, v = (double)(rc / job->W) + 0.5;"),
    "Beer-Lambert adjoint without exp(-I)": ("scale *= exp(-I);", "scale *= 1.0;"),
    "skew sign": ("q[0] = (u - K[1] * q[1] - K[2] * q[2]) / K[0];",
                  "q[0] = (u + K[1] * q[1] - K[2] * q[2]) / K[0];"),
    "slab plane counted as outside": (
        "if (Cijk[a] < lo || Cijk[a] > hi) return 0;", "if (Cijk[a] < lo || Cijk[a] >= hi) return 0;"),
    "clamp instead of zero padding": (
        "if (i < 0 || j < 0 || k < 0 || i >= g->n[0] || j >= g->n[1] || k >= g->n[2]) return 0.0;",
        "if (i < 0) i = 0; if (j < 0) j = 0; if (k < 0) k = 0; if (i >= g->n[0]) i = g->n[0] - 1;"
        " if (j >= g->n[1]) j = g->n[1] - 1; if (k >= g->n[2]) k = g->n[2] - 1;"),
    "spacing ignored in the direction": ("dijk[a] = d[a] / g->spacing[a];", "dijk[a] = d[a];"),
    "bf16 truncation instead of rounding": ("bits += 0x7fffu + lsb;", "(void)lsb;"),
    "alpha pose gradient without the transmittance tangent": (
        "dCv += dT * a * mu + T * da * mu + T * a * dmu;",
        "dCv += T * da * mu + T * a * dmu;"),
    "alpha pose gradient without the step-length tangent": (
        "const double da = (1.0 - a) * (ds * mu + s * dmu);",
        "const double da = (1.0 - a) * (s * dmu);"),
    "pose gradient without the derivative of dt": (
        "grad12[m] = density_factor * (ddt * sum + dt * dsum);",
        "grad12[m] = density_factor * (dt * dsum);"),
    "pose gradient without the unit-length projection": (
        "dd[k] = ((k == c ? 1.0 : 0.0) - dw[k] * dw[c]) * q[r] / nrm;",
        "dd[k] = (k == c ? 1.0 : 0.0) * q[r] / nrm;"),
    "pose gradient exit-plane sign": (
        "dt1 = -(dC[ax1] + t1 * dd[ax1]) / dijk[ax1];", "dt1 = (dC[ax1] + t1 * dd[ax1]) / dijk[ax1];"),
    "pose gradient entry point moving inside the box": (
        "if (!pinned0) dt0 = -(dC[ax0] + t0 * dd[ax0]) / dijk[ax0];",
        "if (ax0 >= 0) dt0 = -(dC[ax0] + t0 * dd[ax0]) / dijk[ax0];"),
    "pose gradient y-derivative sign": (
        "double wy = dj ? f[1] : 1.0 - f[1], sy = dj ? 1.0 : -1.0;",
        "double wy = dj ? f[1] : 1.0 - f[1], sy = dj ? -1.0 : 1.0;"),
    "pose gradient without exp(-I) in Beer-Lambert": (
        "double w = go * (j->mode == ORACLE_BEER_LAMBERT ? exp(-I) : 1.0);", "double w = go;"),
    "alpha colour 1 instead of the intensity": ("out += T * a * mu;", "out += T * a;"),
    "alpha opacity without dt": (
        "double a = -expm1(-density_factor * mu * dt);", "double a = -expm1(-density_factor * mu);"),
    "alpha transmittance not updated": ("T *= 1.0 - a;\n    }\n    return out;",
                                        "(void)T;\n    }\n    return out;"),
    "alpha adjoint transmittance term dropped": (
        "double abar = go * T[i] * mu[i] - Tbar * T[i];", "double abar = go * T[i] * mu[i];"),
    "alpha adjoint direct term dropped": (
        "double mubar = go * T[i] * a[i] + abar * s * (1.0 - a[i]);",
        "double mubar = abar * s * (1.0 - a[i]);"),
    "noise scale sqrt(T i0) instead of sqrt(T / i0)": (
        "double Tn = T > 0.0 ? T + sqrt(T / i0) * z[m] : T;",
        "double Tn = T > 0.0 ? T + sqrt(T * i0) * z[m] : T;"),
    "noise without the upper clamp": ("        if (Tn > 1.0) Tn = 1.0;\n", ""),
    "noise derivative without the 1/2": (
        "if (Tn > 0.0 && Tn < 1.0) slope = 1.0 + z[m] / (2.0 * sqrt(T * i0));",
        "if (Tn > 0.0 && Tn < 1.0) slope = 1.0 + z[m] / sqrt(T * i0);"),
    "siddon cell by floor instead of the nearest centre": (
        "int64_t k = (int64_t)floor(p[a] + 0.5);", "int64_t k = (int64_t)floor(p[a]);"),
    "siddon box of voxel centres instead of cells": (
        "return ray_in_box(g, K, Rt, u, v, 0.5, Cijk, dijk, t0, t1);",
        "return ray_in_box(g, K, Rt, u, v, 0.0, Cijk, dijk, t0, t1);"),
    "siddon crossings unsorted": (
        "qsort(ts + 1, (size_t)(m - 1), sizeof(double), cmp_double);", "(void)cmp_double;"),
    "siddon last interior plane missed": (
        "for (int64_t k = 0; k + 1 < g->n[a]; ++k) {", "for (int64_t k = 0; k + 2 < g->n[a]; ++k) {"),
    "siddon backprojection without density_factor": (
        "double scale = go * density_factor;\n                if (mode == ORACLE_BEER_LAMBERT)\n                    scale *= exp(-ray_siddon",
        "double scale = go;\n                if (mode == ORACLE_BEER_LAMBERT)\n                    scale *= exp(-ray_siddon"),
    "pose gradient translation sign": (
        "for (int k = 0; k < 3; ++k) dC[k] = -Rt[4 * r + k];",
        "for (int k = 0; k < 3; ++k) dC[k] = Rt[4 * r + k];"),
}


PIN_FILES = {"core": "test_oracle_pins.py", "pose": "test_oracle_pose_pins.py",
             "alpha_noise": "test_oracle_alpha_noise_pins.py",
             "siddon": "test_oracle_siddon_pins.py"}


def pin_files_for(name):
    """Every pin file, the mutated part's own first: the run stops at the
    first failing pin (-x), so a mutant fails fast and the suite is the same
    whatever the order."""
    area = ("siddon" if "siddon" in name else "pose" if "pose" in name else
            "alpha_noise" if ("alpha" in name or "noise" in name) else "core")
    order = [area] + [k for k in PIN_FILES if k != area]
    return [os.path.join(ROOT, "tests", PIN_FILES[k]) for k in order]


def run_mutant(name, workdir):
    """Build the oracle with mutant `name` planted and run the pin suite
    against it; returns (returncode, end of its output)."""
    before, after = MUTANTS[name]
    src = open(SRC).read()
    if src.count(before) != 1:
        return None, "mutation site not found: " + name
    tag = "".join(c if c.isalnum() else "_" for c in name)
    c_file = os.path.join(workdir, tag + ".c")
    lib = os.path.join(workdir, tag + ".so")
    with open(c_file, "w") as f:
        f.write(src.replace(before, after))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", lib, c_file, "-lm",
                           "-lpthread"])
    env = dict(os.environ, DRR_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest"] + pin_files_for(name) +
                       ["-q", "-x", "-p", "no:cacheprovider"],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Every mutant's pin run, several at once (each is a separate build and
    interpreter, so they share nothing)."""
    from concurrent.futures import ThreadPoolExecutor
    workdir = str(tmp_path_factory.mktemp("mutants"))
    workers = max(1, min(8, len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(max_workers=workers) as pool:
        futures = {name: pool.submit(run_mutant, name, workdir) for name in MUTANTS}
        return {name: f.result() for name, f in futures.items()}


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, mutant_results):
    code, out = mutant_results[name]
    assert code is not None, out
    assert code != 0, f"mutant '{name}' passed every pin:\n{out}"

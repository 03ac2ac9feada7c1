"""Build libdrr.so (the CUDA path) in-tree with nvcc for sm_100a.

    python -m cone_beam_ct_b200.build [--force]

No fast-math: expm1f / division / sqrt keep their IEEE behaviour.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libdrr.so")
PROBE_LIB = os.path.join(HERE, "libdrr_probe.so")
SOURCES = ["drr_api.cu", "drr_forward.cu", "drr_staged.cu", "drr_adjoint.cu", "drr_prepare.cu",
           "drr_pose.cu", "drr_noise.cu", "drr_siddon.cu"]
HEADERS = ["drr_internal.cuh", "drr_sample.cuh"]
PROBE_SOURCES = ["drr_probe.cu"]
# the same sources with every gather and scatter range-checked (include/drr_debug.h)
CHECKED_LIB = os.path.join(HERE, "libdrr_checked.so")
TEXTURE_LIB = os.path.join(HERE, "libdrr_texture.so")
TEXTURE_SOURCES = ["drr_texture.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "-shared", "-cudart", "shared"]


def _nvcc():
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(home, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib, sources, headers):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in sources + headers]
    deps += [os.path.join(INCLUDE, h)
             for h in ("drr.h", "drr_debug.h", "drr_probe.h", "drr_texture.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def _nvcc_shared(lib, sources, verbose_ptxas, defines=()):
    cmd = [_nvcc()] + ARCH + FLAGS + ["-I", INCLUDE, "-o", lib + ".tmp"]
    cmd += ["-D" + d for d in defines]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in sources]
    subprocess.check_call(cmd)
    os.replace(lib + ".tmp", lib)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Build libdrr.so (the ray-march), libdrr_checked.so (the same with
    every gather and scatter range-checked), libdrr_probe.so (the bench's
    probes) and libdrr_texture.so (the texture-trilinear comparison);
    returns the path of libdrr.so."""
    if force or _stale(LIB, SOURCES, HEADERS):
        _nvcc_shared(LIB, SOURCES, verbose_ptxas)
    if force or _stale(CHECKED_LIB, SOURCES, HEADERS):
        _nvcc_shared(CHECKED_LIB, SOURCES, verbose_ptxas, defines=("DRR_BOUNDS_CHECK",))
    if force or _stale(PROBE_LIB, PROBE_SOURCES, []):
        _nvcc_shared(PROBE_LIB, PROBE_SOURCES, verbose_ptxas)
    if force or _stale(TEXTURE_LIB, TEXTURE_SOURCES, HEADERS):
        _nvcc_shared(TEXTURE_LIB, TEXTURE_SOURCES, verbose_ptxas)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))

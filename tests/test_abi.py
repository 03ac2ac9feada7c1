"""The C ABI on the host (CPU only): libdrr.so loads, exports every entry
point include/drr.h declares, and rejects bad arguments before launching.

Every call here fails host-side validation (or is an empty batch), so no
kernel is ever launched and the fake device addresses are never touched.
"""
import os
import re
import subprocess

import numpy as np
import pytest

from cone_beam_ct_b200 import drr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "drr.h")
PROBE_HEADER = os.path.join(ROOT, "include", "drr_probe.h")
PROBE_LIB = os.path.join(ROOT, "cone_beam_ct_b200", "libdrr_probe.so")
FAKE = 0x7F0000000000          # a plausible device address; never dereferenced here
K_OK = [500.0, 0.0, 99.5, 0.0, 500.0, 99.5, 0.0, 0.0, 1.0]
DIMS, SP, ORG = (16, 16, 16), (1.0, 1.0, 1.0), (0.0, 0.0, 0.0)


def declared_names(header=HEADER, macro="DRR_API"):
    text = open(header).read()
    return sorted(set(re.findall(macro + r"\s+[\w\s\*]+?\b(drr_\w+)\s*\(", text)))


def exported_names(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True,
                         text=True, check=True).stdout
    return set(re.findall(r"\bT\s+(drr_\w+)", out))


def test_header_declares_the_entry_points():
    assert declared_names() == sorted(drr.EXPORTED)


def test_library_exports_every_declared_symbol():
    drr.lib()
    exported = exported_names(drr.LIB_PATH)
    # every declared entry point, and nothing but the ABI, leaves the library
    assert exported == set(declared_names())
    assert drr.drr_abi_version() == 1


def test_checked_library_exports_the_abi_and_its_debug_call():
    checked = os.path.join(ROOT, "cone_beam_ct_b200", "libdrr_checked.so")
    debug = declared_names(os.path.join(ROOT, "include", "drr_debug.h"))
    assert debug == ["drr_debug_bounds_errors"]
    assert exported_names(checked) == set(declared_names()) | set(debug)
    assert "drr_debug_bounds_errors" not in exported_names(drr.LIB_PATH)


def test_checked_library_debug_call_rejects_null_pointers():
    import ctypes
    L = ctypes.CDLL(os.path.join(ROOT, "cone_beam_ct_b200", "libdrr_checked.so"))
    L.drr_debug_bounds_errors.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    L.drr_get_last_error.restype = ctypes.c_char_p
    assert L.drr_debug_bounds_errors(None, None) == drr.DRR_ERR_INVALID_ARG
    assert b"non-NULL" in L.drr_get_last_error()


def test_probe_library_exports_its_declared_symbols():
    import ctypes
    ctypes.CDLL(PROBE_LIB)
    names = declared_names(PROBE_HEADER, "DRR_PROBE_API")
    assert names == ["drr_probe_grid_barrier", "drr_probe_l2_read", "drr_probe_l2_red"]
    assert exported_names(PROBE_LIB) == set(names)


def test_texture_library_exports_its_declared_symbols():
    from cone_beam_ct_b200 import texture
    texture.lib()
    names = declared_names(os.path.join(ROOT, "include", "drr_texture.h"), "DRR_TEX_API")
    assert names == sorted(texture.EXPORTED)
    assert exported_names(texture.LIB_PATH) == set(names)


def test_every_header_is_covered():
    headers = sorted(f for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h"))
    assert headers == ["drr.h", "drr_debug.h", "drr_probe.h", "drr_texture.h"]


def _render(**kw):
    args = dict(vol=FAKE, dtype=drr.DRR_F32, layout=drr.DRR_LAYOUT_LINEAR, dims=DIMS, spacing=SP,
                origin=ORG, K=K_OK, Rt=FAKE, B=2, H=8, W=8, n_samples=16, density_factor=1.0,
                mode=drr.DRR_MODE_RAW, out=FAKE + (1 << 24), stream=0)
    args.update(kw)
    return drr.drr_render(**args)


def _adjoint(**kw):
    args = dict(dims=DIMS, spacing=SP, origin=ORG, K=K_OK, Rt=FAKE, B=2, H=8, W=8,
                n_samples=16, density_factor=1.0, mode=drr.DRR_MODE_RAW,
                grad_out=FAKE + (1 << 20), fwd_out=FAKE + (1 << 21), grad_vol=FAKE + (1 << 24),
                stream=0)
    args.update(kw)
    return drr.drr_render_adjoint(**args)


RENDER_BAD = [
    (dict(dims=(1, 16, 16)), drr.DRR_ERR_INVALID_ARG, "dims"),
    (dict(dims=(16, 16, 1 << 23)), drr.DRR_ERR_INVALID_ARG, "dims"),
    (dict(dims=(2048, 2048, 1024)), drr.DRR_ERR_UNSUPPORTED, "too large"),
    (dict(spacing=(1.0, 0.0, 1.0)), drr.DRR_ERR_INVALID_ARG, "spacing"),
    (dict(spacing=(1.0, float("nan"), 1.0)), drr.DRR_ERR_INVALID_ARG, "spacing"),
    (dict(origin=(0.0, float("inf"), 0.0)), drr.DRR_ERR_INVALID_ARG, "origin"),
    (dict(K=[500.0, 0, 99.5, 1.0, 500.0, 99.5, 0, 0, 1]), drr.DRR_ERR_INVALID_ARG, "triangular"),
    (dict(K=[0.0, 0, 99.5, 0, 500.0, 99.5, 0, 0, 1]), drr.DRR_ERR_INVALID_ARG, "invertible"),
    (dict(K=[500.0, 0, float("nan"), 0, 500.0, 99.5, 0, 0, 1]), drr.DRR_ERR_INVALID_ARG, "finite"),
    (dict(B=-1), drr.DRR_ERR_INVALID_ARG, ">= 0"),
    (dict(B=70000), drr.DRR_ERR_UNSUPPORTED, "views"),
    (dict(H=65535 * 16 + 1), drr.DRR_ERR_UNSUPPORTED, "rows"),
    (dict(n_samples=0), drr.DRR_ERR_INVALID_ARG, "n_samples"),
    (dict(n_samples=(1 << 20) + 1), drr.DRR_ERR_INVALID_ARG, "n_samples"),
    (dict(density_factor=float("inf")), drr.DRR_ERR_INVALID_ARG, "density_factor"),
    (dict(mode=3), drr.DRR_ERR_INVALID_ARG, "mode"),
    (dict(dtype=7), drr.DRR_ERR_INVALID_ARG, "dtype"),
    (dict(layout=5), drr.DRR_ERR_INVALID_ARG, "layout"),
    (dict(vol=0), drr.DRR_ERR_INVALID_ARG, "vol"),
    (dict(vol=FAKE + 2), drr.DRR_ERR_INVALID_ARG, "vol"),       # fp32 volume, 2-byte aligned
    (dict(Rt=0), drr.DRR_ERR_INVALID_ARG, "Rt"),
    (dict(Rt=FAKE + 1), drr.DRR_ERR_INVALID_ARG, "Rt"),
    (dict(out=0), drr.DRR_ERR_INVALID_ARG, "out"),
    (dict(layout=drr.DRR_LAYOUT_CORNERS, vol=FAKE + 4), drr.DRR_ERR_INVALID_ARG, "16 bytes"),
    (dict(layout=drr.DRR_LAYOUT_QUADS, vol=FAKE + 8), drr.DRR_ERR_INVALID_ARG, "16 bytes"),
    (dict(out=FAKE + 6), drr.DRR_ERR_INVALID_ARG, "out"),
]


@pytest.mark.parametrize("kw,status,word", RENDER_BAD)
def test_render_rejects_bad_arguments(kw, status, word):
    with pytest.raises(drr.DrrError) as e:
        _render(**kw)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


ADJOINT_BAD = [
    (dict(dims=(16, 0, 16)), drr.DRR_ERR_INVALID_ARG),
    (dict(n_samples=-3), drr.DRR_ERR_INVALID_ARG),
    (dict(grad_out=0), drr.DRR_ERR_INVALID_ARG),
    (dict(grad_vol=0), drr.DRR_ERR_INVALID_ARG),
    (dict(mode=drr.DRR_MODE_BEER_LAMBERT, fwd_out=0), drr.DRR_ERR_INVALID_ARG),
    (dict(grad_vol=FAKE + (1 << 20)), drr.DRR_ERR_INVALID_ARG),    # overlaps grad_out
    (dict(K=[500.0, 0, 99.5, 0, 500.0, 99.5, 0.5, 0, 1]), drr.DRR_ERR_INVALID_ARG),
    (dict(mode=-1), drr.DRR_ERR_INVALID_ARG),
    (dict(mode=drr.DRR_MODE_ALPHA), drr.DRR_ERR_UNSUPPORTED),      # needs the volume
]


def _staged(**kw):
    args = dict(vol=FAKE, dtype=drr.DRR_F32, dims=DIMS, spacing=SP, origin=ORG, K=K_OK,
                Rt=FAKE + (1 << 26), B=2, H=8, W=8, n_samples=16, density_factor=1.0,
                mode=drr.DRR_MODE_RAW, out=FAKE + (1 << 27), stream=0)
    args.update(kw)
    return drr.drr_render_staged(**args)


STAGED_BAD = [
    (dict(vol=0), drr.DRR_ERR_INVALID_ARG, "vol"),
    (dict(vol=FAKE + 8), drr.DRR_ERR_INVALID_ARG, "16-byte"),
    (dict(out=0), drr.DRR_ERR_INVALID_ARG, "out"),
    (dict(mode=drr.DRR_MODE_ALPHA), drr.DRR_ERR_UNSUPPORTED, "alpha"),
    (dict(dtype=7), drr.DRR_ERR_INVALID_ARG, "dtype"),
    (dict(n_samples=0), drr.DRR_ERR_INVALID_ARG, "n_samples"),
    (dict(dims=(1, 16, 16)), drr.DRR_ERR_INVALID_ARG, "dims"),
]


@pytest.mark.parametrize("kw,status,word", STAGED_BAD)
def test_staged_render_rejects_bad_arguments(kw, status, word):
    with pytest.raises(drr.DrrError) as e:
        _staged(**kw)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


def test_staged_render_empty_batch_is_a_no_op():
    _staged(B=0, vol=None, out=None, Rt=None)
    assert drr.drr_get_last_error() == ""


@pytest.mark.parametrize("kw,status", ADJOINT_BAD)
def test_adjoint_rejects_bad_arguments(kw, status):
    with pytest.raises(drr.DrrError) as e:
        _adjoint(**kw)
    assert e.value.status == status


WS = FAKE + (1 << 30)
WS_BYTES = 1 << 28


def _adjoint_ws(**kw):
    args = dict(dims=DIMS, spacing=SP, origin=ORG, K=K_OK, Rt=FAKE, B=2, H=8, W=8,
                n_samples=16, density_factor=1.0, mode=drr.DRR_MODE_RAW,
                grad_out=FAKE + (1 << 20), fwd_out=None, grad_vol=FAKE + (1 << 24),
                workspace=WS, workspace_bytes=WS_BYTES, stream=0)
    args.update(kw)
    return drr.drr_render_adjoint_ws(**args)


WS_BAD = [
    (dict(workspace=0), "workspace"),
    (dict(workspace=WS + 16), "aligned"),
    (dict(workspace_bytes=100), "needed"),
    (dict(workspace=FAKE + (1 << 24)), "overlaps"),          # on grad_vol
    (dict(n_samples=0), "n_samples"),
]


@pytest.mark.parametrize("kw,word", WS_BAD)
def test_workspace_adjoint_rejects_bad_arguments(kw, word):
    with pytest.raises(drr.DrrError) as e:
        _adjoint_ws(**kw)
    assert e.value.status == drr.DRR_ERR_INVALID_ARG
    assert word in drr.drr_get_last_error()


def ws_header(B):
    """Adjoint workspace header for B output images: 1 + B int flags; 16
    bytes of barrier words (16-byte aligned); B views of 96 bytes (256-byte
    aligned); the records then start 256-byte aligned."""
    up = lambda n, a: (n + a - 1) // a * a
    bar = up((1 + B) * 4, 16)
    views = up(bar + 16, 256)
    return up(views + 96 * B, 256)


def test_workspace_bytes():
    assert ws_header(2) == 512 and ws_header(64) == 6656
    assert drr.drr_adjoint_workspace_bytes((16, 16, 16), 2) == ws_header(2) + 15 ** 3 * 32
    assert drr.drr_adjoint_workspace_bytes((256, 256, 256), 64) == ws_header(64) + 255 ** 3 * 32
    assert drr.drr_adjoint_workspace_bytes((1, 16, 16), 2) == 0
    assert drr.drr_adjoint_workspace_bytes((16, 16, 16), -1) == 0
    _adjoint_ws(B=0, workspace=None, grad_out=None, grad_vol=None, Rt=None)   # empty: no-op


def _adjoint_noalloc(**kw):
    args = dict(dims=DIMS, spacing=SP, origin=ORG, K=K_OK, Rt=FAKE, B=2, H=8, W=8,
                n_samples=16, density_factor=1.0, mode=drr.DRR_MODE_RAW,
                grad_out=FAKE + (1 << 20), fwd_out=None, grad_vol=FAKE + (1 << 24), stream=0)
    args.update(kw)
    return drr.drr_render_adjoint_noalloc(**args)


# every one of these is rejected before the built-in scratch's address is
# looked up, so nothing touches a device
NOALLOC_BAD = [
    (dict(grad_out=0), drr.DRR_ERR_INVALID_ARG, "grad_out"),
    (dict(grad_vol=FAKE + (1 << 24) + 2), drr.DRR_ERR_INVALID_ARG, "grad_vol"),
    (dict(mode=drr.DRR_MODE_BEER_LAMBERT, fwd_out=None), drr.DRR_ERR_INVALID_ARG, "fwd_out"),
    (dict(grad_vol=FAKE + (1 << 20) + 64), drr.DRR_ERR_INVALID_ARG, "overlaps"),
    (dict(mode=drr.DRR_MODE_BEER_LAMBERT, fwd_out=FAKE + (1 << 24)), drr.DRR_ERR_INVALID_ARG,
     "overlaps"),
    (dict(mode=drr.DRR_MODE_ALPHA), drr.DRR_ERR_UNSUPPORTED, "ALPHA"),
    (dict(n_samples=0), drr.DRR_ERR_INVALID_ARG, "n_samples"),
    (dict(dims=(1, 16, 16)), drr.DRR_ERR_INVALID_ARG, "dims"),
    (dict(dims=(128, 128, 128), grad_vol=FAKE + (1 << 32)), drr.DRR_ERR_UNSUPPORTED,
     "built-in scratch"),
]


@pytest.mark.parametrize("kw,status,word", NOALLOC_BAD)
def test_noalloc_adjoint_rejects_bad_arguments(kw, status, word):
    with pytest.raises(drr.DrrError) as e:
        _adjoint_noalloc(**kw)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


def test_noalloc_adjoint_empty_batch_is_a_no_op():
    _adjoint_noalloc(B=0, grad_out=None, grad_vol=None, Rt=None)
    assert drr.drr_get_last_error() == ""


def test_noalloc_scratch_size_is_the_headers():
    m = re.search(r"#define\s+DRR_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)",
                  open(HEADER).read())
    assert m, "DRR_NOALLOC_SCRATCH_BYTES not found in include/drr.h"
    assert drr.DRR_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_raw_adjoint_does_not_need_the_forward_image():
    # fwd_out may be NULL in RAW mode: only an empty batch keeps this off the device
    _adjoint(fwd_out=None, B=0)


@pytest.mark.parametrize("which", ["B", "H", "W"])
def test_empty_batch_or_image_is_a_no_op(which):
    # nothing to launch: succeeds even with NULL buffers
    _render(**{which: 0, "vol": None, "out": None, "Rt": None})
    _adjoint(**{which: 0, "grad_out": None, "grad_vol": None, "Rt": None, "fwd_out": None})
    assert drr.drr_get_last_error() == ""


def _pose(**kw):
    args = dict(vol=FAKE, dtype=drr.DRR_F32, layout=drr.DRR_LAYOUT_LINEAR, dims=DIMS, spacing=SP,
                origin=ORG, K=K_OK, Rt=FAKE + (1 << 26), B=2, H=8, W=8, n_samples=16,
                density_factor=1.0, mode=drr.DRR_MODE_RAW, grad_out=FAKE + (1 << 20),
                fwd_out=FAKE + (1 << 21), grad_Rt=FAKE + (1 << 27), stream=0)
    args.update(kw)
    return drr.drr_render_pose_grad(**args)


POSE_BAD = [
    (dict(dims=(16, 1, 16)), drr.DRR_ERR_INVALID_ARG, "dims"),
    (dict(mode=3), drr.DRR_ERR_INVALID_ARG, "mode"),
    (dict(layout=9), drr.DRR_ERR_INVALID_ARG, "layout"),
    (dict(vol=0), drr.DRR_ERR_INVALID_ARG, "vol"),
    (dict(layout=drr.DRR_LAYOUT_CORNERS, vol=FAKE + 8), drr.DRR_ERR_INVALID_ARG, "16 bytes"),
    (dict(grad_out=0), drr.DRR_ERR_INVALID_ARG, "grad_out"),
    (dict(mode=drr.DRR_MODE_BEER_LAMBERT, fwd_out=0), drr.DRR_ERR_INVALID_ARG, "fwd_out"),
    (dict(grad_Rt=0), drr.DRR_ERR_INVALID_ARG, "grad_Rt"),
    (dict(grad_Rt=FAKE + (1 << 26) + 8), drr.DRR_ERR_INVALID_ARG, "overlaps"),   # on Rt
    (dict(grad_Rt=FAKE + (1 << 20) + 4), drr.DRR_ERR_INVALID_ARG, "overlaps"),   # on grad_out
    (dict(n_samples=0), drr.DRR_ERR_INVALID_ARG, "n_samples"),
    (dict(mode=drr.DRR_MODE_ALPHA, fwd_out=0), drr.DRR_ERR_INVALID_ARG, "alpha"),
]


@pytest.mark.parametrize("kw,status,word", POSE_BAD)
def test_pose_gradient_rejects_bad_arguments(kw, status, word):
    with pytest.raises(drr.DrrError) as e:
        _pose(**kw)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


def test_pose_gradient_empty_batch_is_a_no_op():
    _pose(B=0, vol=None, grad_out=None, fwd_out=None, grad_Rt=None, Rt=None)
    assert drr.drr_get_last_error() == ""


def _alpha_adjoint(**kw):
    args = dict(vol=FAKE, dtype=drr.DRR_F32, layout=drr.DRR_LAYOUT_LINEAR, dims=DIMS, spacing=SP,
                origin=ORG, K=K_OK, Rt=FAKE + (1 << 26), B=2, H=8, W=8, n_samples=16,
                density_factor=1.0, grad_out=FAKE + (1 << 20), fwd_out=FAKE + (1 << 21),
                grad_vol=FAKE + (1 << 24), stream=0)
    args.update(kw)
    return drr.drr_render_alpha_adjoint(**args)


ALPHA_BAD = [
    (dict(layout=drr.DRR_LAYOUT_PADDED), drr.DRR_ERR_UNSUPPORTED, "LINEAR"),
    (dict(fwd_out=0), drr.DRR_ERR_INVALID_ARG, "alpha image"),
    (dict(grad_out=0), drr.DRR_ERR_INVALID_ARG, "grad_out"),
    (dict(grad_vol=0), drr.DRR_ERR_INVALID_ARG, "grad_vol"),
    (dict(vol=0), drr.DRR_ERR_INVALID_ARG, "vol"),
    (dict(grad_vol=FAKE), drr.DRR_ERR_INVALID_ARG, "overlaps"),        # on the volume
    (dict(dims=(16, 16, 0)), drr.DRR_ERR_INVALID_ARG, "dims"),
]


@pytest.mark.parametrize("kw,status,word", ALPHA_BAD)
def test_alpha_adjoint_rejects_bad_arguments(kw, status, word):
    with pytest.raises(drr.DrrError) as e:
        _alpha_adjoint(**kw)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


def _alpha_adjoint_ws(**kw):
    args = dict(vol=FAKE, dtype=drr.DRR_F32, layout=drr.DRR_LAYOUT_LINEAR, dims=DIMS, spacing=SP,
                origin=ORG, K=K_OK, Rt=FAKE + (1 << 26), B=2, H=8, W=8, n_samples=16,
                density_factor=1.0, grad_out=FAKE + (1 << 20), fwd_out=FAKE + (1 << 21),
                grad_vol=FAKE + (1 << 24), workspace=WS, workspace_bytes=WS_BYTES, stream=0)
    args.update(kw)
    return drr.drr_render_alpha_adjoint_ws(**args)


ALPHA_WS_BAD = [
    (dict(workspace=0), drr.DRR_ERR_INVALID_ARG, "workspace"),
    (dict(workspace=WS + 16), drr.DRR_ERR_INVALID_ARG, "aligned"),
    (dict(workspace_bytes=100), drr.DRR_ERR_INVALID_ARG, "needed"),
    (dict(workspace=FAKE), drr.DRR_ERR_INVALID_ARG, "overlaps"),             # on the volume
    (dict(workspace=FAKE + (1 << 21)), drr.DRR_ERR_INVALID_ARG, "overlaps"),  # on fwd_out
    (dict(layout=drr.DRR_LAYOUT_PADDED), drr.DRR_ERR_UNSUPPORTED, "LINEAR"),
    (dict(fwd_out=0), drr.DRR_ERR_INVALID_ARG, "alpha image"),
]


@pytest.mark.parametrize("kw,status,word", ALPHA_WS_BAD)
def test_alpha_adjoint_ws_rejects_bad_arguments(kw, status, word):
    with pytest.raises(drr.DrrError) as e:
        _alpha_adjoint_ws(**kw)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


def test_alpha_adjoint_ws_empty_batch_is_a_no_op():
    _alpha_adjoint_ws(B=0, vol=None, workspace=None, grad_out=None, fwd_out=None, grad_vol=None,
                      Rt=None)
    assert drr.drr_get_last_error() == ""


NOISE_BAD = [
    (dict(i0=0.0), "i0"),
    (dict(i0=float("inf")), "i0"),
    (dict(n=-1), "n must"),
    (dict(z=0), "non-NULL"),
    (dict(out=FAKE + 4), "overlaps"),          # part of image
    (dict(out=FAKE + (1 << 20)), "overlaps"),  # z
]


@pytest.mark.parametrize("kw,word", NOISE_BAD)
def test_noise_rejects_bad_arguments(kw, word):
    args = dict(image=FAKE, z=FAKE + (1 << 20), i0=100.0, out=FAKE + (1 << 21), n=1000, stream=0)
    args.update(kw)
    with pytest.raises(drr.DrrError) as e:
        drr.drr_poisson_noise(**args)
    assert e.value.status == drr.DRR_ERR_INVALID_ARG
    assert word in drr.drr_get_last_error()


def test_noise_backward_rejects_bad_arguments():
    args = dict(image=FAKE, z=FAKE + (1 << 20), i0=100.0, grad_out=FAKE + (1 << 21),
                grad_image=FAKE + (1 << 22), n=1000, stream=0)
    for kw in (dict(i0=-1.0), dict(grad_image=FAKE + 8), dict(grad_out=0)):
        with pytest.raises(drr.DrrError) as e:
            drr.drr_poisson_noise_backward(**dict(args, **kw))
        assert e.value.status == drr.DRR_ERR_INVALID_ARG
    drr.drr_poisson_noise(FAKE, FAKE, 1.0, FAKE, n=0, stream=0)           # empty: no-op
    drr.drr_poisson_noise_backward(FAKE, FAKE, 1.0, FAKE, FAKE, n=0, stream=0)


SIDDON_BAD = [
    (dict(mode=drr.DRR_MODE_ALPHA), drr.DRR_ERR_UNSUPPORTED, "RAW"),
    (dict(mode=5), drr.DRR_ERR_INVALID_ARG, "mode"),
    (dict(dtype=4), drr.DRR_ERR_INVALID_ARG, "dtype"),
    (dict(vol=0), drr.DRR_ERR_INVALID_ARG, "vol"),
    (dict(out=0), drr.DRR_ERR_INVALID_ARG, "out"),
    (dict(dims=(16, 1, 16)), drr.DRR_ERR_INVALID_ARG, "dims"),
    (dict(density_factor=float("nan")), drr.DRR_ERR_INVALID_ARG, "density_factor"),
]


@pytest.mark.parametrize("kw,status,word", SIDDON_BAD)
def test_siddon_rejects_bad_arguments(kw, status, word):
    args = dict(vol=FAKE, dtype=drr.DRR_F32, dims=DIMS, spacing=SP, origin=ORG, K=K_OK, Rt=FAKE,
                B=2, H=8, W=8, density_factor=1.0, mode=drr.DRR_MODE_RAW, out=FAKE + (1 << 20),
                stream=0)
    args.update(kw)
    with pytest.raises(drr.DrrError) as e:
        drr.drr_render_siddon(**args)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


def test_siddon_adjoint_rejects_bad_arguments():
    args = dict(dims=DIMS, spacing=SP, origin=ORG, K=K_OK, Rt=FAKE, B=2, H=8, W=8,
                density_factor=1.0, mode=drr.DRR_MODE_RAW, grad_out=FAKE + (1 << 20),
                fwd_out=None, grad_vol=FAKE + (1 << 24), stream=0)
    for kw, status in ((dict(grad_out=0), drr.DRR_ERR_INVALID_ARG),
                       (dict(mode=drr.DRR_MODE_BEER_LAMBERT), drr.DRR_ERR_INVALID_ARG),
                       (dict(grad_vol=FAKE + (1 << 20) + 4), drr.DRR_ERR_INVALID_ARG),
                       (dict(mode=drr.DRR_MODE_ALPHA), drr.DRR_ERR_UNSUPPORTED)):
        with pytest.raises(drr.DrrError) as e:
            drr.drr_render_siddon_adjoint(**dict(args, **kw))
        assert e.value.status == status
    drr.drr_render_siddon_adjoint(**dict(args, B=0, grad_out=None, grad_vol=None))   # no-op


def test_batched_rejects_bad_arguments():
    args = dict(vols=FAKE, dtype=drr.DRR_F32, layout=drr.DRR_LAYOUT_LINEAR, dims=DIMS, spacing=SP,
                origin=ORG, K=K_OK, Rt=FAKE + (1 << 26), n_vols=2, channels=3, n_views=4, H=8, W=8,
                n_samples=16, density_factor=1.0, mode=drr.DRR_MODE_RAW, out=FAKE + (1 << 20),
                stream=0)
    for kw, status, word in ((dict(n_views=3), drr.DRR_ERR_INVALID_ARG, "multiple"),
                             (dict(channels=-1), drr.DRR_ERR_INVALID_ARG, ">= 0"),
                             (dict(channels=20000), drr.DRR_ERR_UNSUPPORTED, "images"),
                             (dict(vols=0), drr.DRR_ERR_INVALID_ARG, "vols"),
                             (dict(out=0), drr.DRR_ERR_INVALID_ARG, "out")):
        with pytest.raises(drr.DrrError) as e:
            drr.drr_render_batched(**dict(args, **kw))
        assert e.value.status == status and word in drr.drr_get_last_error()
    drr.drr_render_batched(**dict(args, channels=0, vols=None, out=None))   # empty: no-op
    adj = dict(dims=DIMS, spacing=SP, origin=ORG, K=K_OK, Rt=FAKE, n_vols=2, channels=1,
               n_views=1, H=8, W=8, n_samples=16, density_factor=1.0, mode=drr.DRR_MODE_RAW,
               grad_out=FAKE + (1 << 20), fwd_out=None, grad_vols=FAKE + (1 << 24), stream=0)
    for kw in (dict(grad_out=0), dict(n_views=5), dict(mode=drr.DRR_MODE_BEER_LAMBERT),
               dict(grad_vols=FAKE + (1 << 20) + 4)):
        with pytest.raises(drr.DrrError):
            drr.drr_render_adjoint_batched(**dict(adj, **kw))


def test_batched_workspace_bytes():
    # the header of one output image per (view, channel) -- 4 x 3 images; 2
    # x 3 when one view is broadcast to both volumes -- then 32 bytes per
    # cell for each of the n_vols * channels volume-channels
    assert drr.drr_adjoint_batched_workspace_bytes((16, 16, 16), 2, 3, 4) == \
        ws_header(12) + 6 * 15 ** 3 * 32
    assert drr.drr_adjoint_batched_workspace_bytes((16, 16, 16), 2, 3, 1) == \
        ws_header(6) + 6 * 15 ** 3 * 32
    assert drr.drr_adjoint_batched_workspace_bytes((16, 16, 16), 1, 1, 64) == \
        drr.drr_adjoint_workspace_bytes((16, 16, 16), 64)
    assert drr.drr_adjoint_batched_workspace_bytes((16, 16, 16), 2, 3, 3) == 0   # 3 % 2 != 0
    assert drr.drr_adjoint_batched_workspace_bytes((16, 16, 16), 0, 3, 4) == 0
    assert drr.drr_adjoint_batched_workspace_bytes((1, 16, 16), 2, 3, 4) == 0
    assert drr.drr_adjoint_batched_workspace_bytes((16, 16, 16), 1, 2, 40000) == 0


def _adjoint_batched_ws(**kw):
    args = dict(dims=DIMS, spacing=SP, origin=ORG, K=K_OK, Rt=FAKE, n_vols=2, channels=1,
                n_views=2, H=8, W=8, n_samples=16, density_factor=1.0, mode=drr.DRR_MODE_RAW,
                grad_out=FAKE + (1 << 20), fwd_out=None, grad_vols=FAKE + (1 << 24),
                workspace=WS, workspace_bytes=WS_BYTES, stream=0)
    args.update(kw)
    return drr.drr_render_adjoint_batched_ws(**args)


BATCHED_WS_BAD = [
    (dict(workspace=0), "workspace"),
    (dict(workspace=WS + 64), "aligned"),
    (dict(workspace_bytes=1000), "needed"),
    (dict(workspace=FAKE + (1 << 24)), "overlaps"),          # on grad_vols
    (dict(n_views=3), "multiple"),
]


@pytest.mark.parametrize("kw,word", BATCHED_WS_BAD)
def test_batched_workspace_adjoint_rejects_bad_arguments(kw, word):
    with pytest.raises(drr.DrrError) as e:
        _adjoint_batched_ws(**kw)
    assert e.value.status == drr.DRR_ERR_INVALID_ARG
    assert word in drr.drr_get_last_error()


def _pose_batched(**kw):
    args = dict(vols=FAKE, dtype=drr.DRR_F32, layout=drr.DRR_LAYOUT_LINEAR, dims=DIMS, spacing=SP,
                origin=ORG, K=K_OK, Rt=FAKE + (1 << 26), n_vols=2, channels=2, n_views=4, H=8,
                W=8, n_samples=16, density_factor=1.0, mode=drr.DRR_MODE_RAW,
                grad_out=FAKE + (1 << 20), fwd_out=None, grad_Rt=FAKE + (1 << 27), stream=0)
    args.update(kw)
    return drr.drr_render_pose_grad_batched(**args)


POSE_BATCHED_BAD = [
    (dict(n_views=3), drr.DRR_ERR_INVALID_ARG, "multiple"),
    (dict(mode=drr.DRR_MODE_ALPHA), drr.DRR_ERR_INVALID_ARG, "fwd_out"),
    (dict(mode=drr.DRR_MODE_BEER_LAMBERT), drr.DRR_ERR_INVALID_ARG, "fwd_out"),
    (dict(grad_Rt=0), drr.DRR_ERR_INVALID_ARG, "grad_Rt"),
    (dict(grad_Rt=FAKE + (1 << 26)), drr.DRR_ERR_INVALID_ARG, "overlaps"),   # on Rt
    (dict(vols=0), drr.DRR_ERR_INVALID_ARG, "vols"),
    (dict(layout=drr.DRR_LAYOUT_QUADS, vols=FAKE + 8), drr.DRR_ERR_INVALID_ARG, "16 bytes"),
]


@pytest.mark.parametrize("kw,status,word", POSE_BATCHED_BAD)
def test_batched_pose_gradient_rejects_bad_arguments(kw, status, word):
    with pytest.raises(drr.DrrError) as e:
        _pose_batched(**kw)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


def test_batched_pose_gradient_empty_batch_is_a_no_op():
    _pose_batched(channels=0, vols=None, grad_out=None, grad_Rt=None)
    assert drr.drr_get_last_error() == ""


def _alpha_batched(**kw):
    args = dict(vols=FAKE, dtype=drr.DRR_F32, layout=drr.DRR_LAYOUT_CORNERS, dims=DIMS, spacing=SP,
                origin=ORG, K=K_OK, Rt=FAKE + (1 << 26), n_vols=2, channels=1, n_views=2, H=8,
                W=8, n_samples=16, density_factor=1.0, grad_out=FAKE + (1 << 27),
                fwd_out=FAKE + (1 << 28), grad_vols=FAKE + (1 << 29), workspace=None, stream=0)
    args.update(kw)
    return drr.drr_render_alpha_adjoint_batched(**args)


ALPHA_BATCHED_BAD = [
    (dict(layout=drr.DRR_LAYOUT_PADDED), drr.DRR_ERR_UNSUPPORTED, "LINEAR"),
    (dict(fwd_out=0), drr.DRR_ERR_INVALID_ARG, "alpha image"),
    (dict(n_views=3), drr.DRR_ERR_INVALID_ARG, "multiple"),
    (dict(grad_vols=FAKE), drr.DRR_ERR_INVALID_ARG, "overlaps"),          # on the volumes
    (dict(workspace=WS, workspace_bytes=1000), drr.DRR_ERR_INVALID_ARG, "needed"),
    (dict(workspace=WS + 64, workspace_bytes=WS_BYTES), drr.DRR_ERR_INVALID_ARG, "aligned"),
]


@pytest.mark.parametrize("kw,status,word", ALPHA_BATCHED_BAD)
def test_batched_alpha_adjoint_rejects_bad_arguments(kw, status, word):
    with pytest.raises(drr.DrrError) as e:
        _alpha_batched(**kw)
    assert e.value.status == status
    assert word in drr.drr_get_last_error()


def test_prepared_bytes():
    assert drr.drr_prepared_bytes((256, 256, 256), drr.DRR_F32, drr.DRR_LAYOUT_LINEAR) == 4 * 256 ** 3
    assert drr.drr_prepared_bytes((256, 256, 256), drr.DRR_BF16, drr.DRR_LAYOUT_LINEAR) == 2 * 256 ** 3
    assert drr.drr_prepared_bytes((5, 6, 7), drr.DRR_F32, drr.DRR_LAYOUT_PADDED) == 4 * 7 * 8 * 9
    assert drr.drr_prepared_bytes((5, 6, 7), drr.DRR_BF16, drr.DRR_LAYOUT_PADDED) == 2 * 7 * 8 * 9
    assert drr.drr_prepared_bytes((1, 6, 7), drr.DRR_F32, drr.DRR_LAYOUT_PADDED) == 0
    assert drr.drr_prepared_bytes((5, 6, 7), 3, drr.DRR_LAYOUT_PADDED) == 0
    assert drr.drr_prepared_bytes((2048, 2048, 1024), drr.DRR_F32, drr.DRR_LAYOUT_LINEAR) == 0
    assert drr.drr_prepared_bytes((5, 6, 7), drr.DRR_F32, drr.DRR_LAYOUT_CORNERS) == 4 * 8 * 4 * 5 * 6
    assert drr.drr_prepared_bytes((5, 6, 7), drr.DRR_BF16, drr.DRR_LAYOUT_CORNERS) == 2 * 8 * 4 * 5 * 6
    assert drr.drr_prepared_bytes((640, 640, 640), drr.DRR_BF16, drr.DRR_LAYOUT_CORNERS) == 2 * 8 * 639 ** 3
    assert drr.drr_prepared_bytes((660, 660, 660), drr.DRR_BF16, drr.DRR_LAYOUT_CORNERS) == 0
    assert drr.drr_prepared_bytes((5, 6, 7), drr.DRR_F32, drr.DRR_LAYOUT_QUADS) == 4 * 4 * 4 * 5 * 7
    assert drr.drr_prepared_bytes((5, 6, 7), drr.DRR_BF16, drr.DRR_LAYOUT_QUADS) == 2 * 4 * 4 * 5 * 7
    assert drr.drr_prepared_bytes((1024, 1024, 512), drr.DRR_F32, drr.DRR_LAYOUT_QUADS) == \
        4 * 4 * 1023 * 1023 * 512
    # bricks of 8^3 cells, 736 elements each: ceil((n - 1) / 8) per axis
    assert drr.drr_prepared_bytes((256, 256, 256), drr.DRR_F32, drr.DRR_LAYOUT_BRICKS) == \
        4 * 736 * 32 ** 3
    assert drr.drr_prepared_bytes((9, 10, 17), drr.DRR_BF16, drr.DRR_LAYOUT_BRICKS) == \
        2 * 736 * 1 * 2 * 2
    assert drr.drr_prepared_bytes((2, 2, 2), drr.DRR_F32, drr.DRR_LAYOUT_BRICKS) == 4 * 736


PREPARE_BAD = [
    (dict(dims=(16, 16, 1)), drr.DRR_ERR_INVALID_ARG),
    (dict(dtype=4), drr.DRR_ERR_INVALID_ARG),
    (dict(layout=9), drr.DRR_ERR_INVALID_ARG),
    (dict(src=0), drr.DRR_ERR_INVALID_ARG),
    (dict(dst=0), drr.DRR_ERR_INVALID_ARG),
    (dict(dst_bytes=100), drr.DRR_ERR_INVALID_ARG),
    (dict(dst=FAKE + 64), drr.DRR_ERR_INVALID_ARG),      # overlaps src
    (dict(src=FAKE + 2), drr.DRR_ERR_INVALID_ARG),       # misaligned
    (dict(layout=drr.DRR_LAYOUT_CORNERS, dst=FAKE + (1 << 24) + 8), drr.DRR_ERR_INVALID_ARG),
    (dict(layout=drr.DRR_LAYOUT_QUADS, dst=FAKE + (1 << 24) + 8), drr.DRR_ERR_INVALID_ARG),
    (dict(layout=drr.DRR_LAYOUT_BRICKS, dst=FAKE + (1 << 24) + 8), drr.DRR_ERR_INVALID_ARG),
    (dict(dims=(2048, 2048, 1024)), drr.DRR_ERR_UNSUPPORTED),
]


@pytest.mark.parametrize("kw,status", PREPARE_BAD)
def test_prepare_rejects_bad_arguments(kw, status):
    args = dict(src=FAKE, dims=DIMS, dtype=drr.DRR_BF16, layout=drr.DRR_LAYOUT_PADDED,
                dst=FAKE + (1 << 24), dst_bytes=1 << 24, stream=0)
    args.update(kw)
    with pytest.raises(drr.DrrError) as e:
        drr.drr_prepare_volume(**args)
    assert e.value.status == status


def test_binding_refuses_host_tensors_for_device_arguments():
    torch = pytest.importorskip("torch")
    with pytest.raises(TypeError):
        _render(out=torch.zeros(2, 8, 8))


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(drr, "_lib", None)
    monkeypatch.setattr(drr, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        drr.lib()


def test_grid_barrier_probe_rejects_bad_arguments():
    # no GPU needed: argument checks come before any CUDA call
    import ctypes
    lib = ctypes.CDLL(PROBE_LIB)
    f = lib.drr_probe_grid_barrier
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p]
    f.restype = ctypes.c_int
    t, p, c = ctypes.c_ulonglong(), ctypes.c_int(), ctypes.c_int()
    ok = (ctypes.byref(t), ctypes.byref(p), ctypes.byref(c))
    assert f(-1, 1, 10.0, *ok) == -1
    assert f(0, 0, 10.0, *ok) == -1
    assert f(0, 5000, 10.0, *ok) == -1
    assert f(0, 1, 0.0, *ok) == -1
    assert f(0, 1, 1e9, *ok) == -1
    assert f(0, 1, 10.0, None, ok[1], ok[2]) == -1

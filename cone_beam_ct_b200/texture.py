"""Binding of libdrr_texture.so: the texture-trilinear comparison path
(include/drr_texture.h) -- not the product path.  Argument marshalling only.
"""
import ctypes
import os

from .drr import _dev, _f3v, _f9v, _i3v, _stream

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdrr_texture.so")
EXPORTED = ("drr_tex_create", "drr_tex_render", "drr_tex_destroy", "drr_tex_last_error")
TEXEL_F32, TEXEL_F16 = 0, 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdrr_texture.so is not built ({LIB_PATH})")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.drr_tex_create.argtypes = [vp, ctypes.c_int * 3, ci, ctypes.POINTER(vp)]
        L.drr_tex_create.restype = ci
        L.drr_tex_render.argtypes = [vp, ctypes.c_float * 3, ctypes.c_float * 3,
                                     ctypes.c_float * 9, vp, ci, ci, ci, ci, cf, ci, vp, vp]
        L.drr_tex_render.restype = ci
        L.drr_tex_destroy.argtypes = [vp]
        L.drr_tex_destroy.restype = ci
        L.drr_tex_last_error.argtypes = []
        L.drr_tex_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"libdrr_texture rc {rc}: {lib().drr_tex_last_error().decode()}")


class TextureVolume:
    """A volume copied into a 3-D texture (float32 or float16 texels)."""

    def __init__(self, vol, dims, texel=TEXEL_F32):
        h = ctypes.c_void_p()
        _check(lib().drr_tex_create(_dev(vol, "vol"), _i3v(dims), int(texel), ctypes.byref(h)))
        self.handle = h

    def render(self, spacing, origin, K, Rt, B, H, W, n_samples, density_factor, mode, out,
               stream=None):
        _check(lib().drr_tex_render(self.handle, _f3v(spacing), _f3v(origin), _f9v(K),
                                    _dev(Rt, "Rt"), int(B), int(H), int(W), int(n_samples),
                                    float(density_factor), int(mode), _dev(out, "out"),
                                    _stream(stream)))

    def close(self):
        if self.handle:
            _check(lib().drr_tex_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

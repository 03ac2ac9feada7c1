"""Python binding of libdrr.so: the C ABI of include/drr.h, same names.

Argument marshalling only -- every step of the ray-march runs in the CUDA
kernels of libdrr.so.  Device arguments are CUDA tensors (or raw device
addresses as int); host arguments (dims, spacing, origin, K) are sequences
or numpy arrays.  ``stream`` defaults to torch's current CUDA stream.  A
non-OK status raises DrrError with the library's own message.  If the
library has not been built, every call raises: there is no fallback.
"""
import ctypes
import os

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdrr.so")
# the bounds-checked debug build of the same sources (include/drr_debug.h)
CHECKED_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdrr_checked.so")

DRR_OK, DRR_ERR_INVALID_ARG, DRR_ERR_UNSUPPORTED, DRR_ERR_CUDA = 0, 1, 2, 3
DRR_MODE_RAW, DRR_MODE_BEER_LAMBERT, DRR_MODE_ALPHA = 0, 1, 2
DRR_F32, DRR_BF16 = 0, 1
DRR_LAYOUT_LINEAR, DRR_LAYOUT_PADDED, DRR_LAYOUT_CORNERS, DRR_LAYOUT_QUADS = 0, 1, 2, 3
DRR_LAYOUT_BRICKS = 4

# names exported by libdrr.so (include/drr.h)
EXPORTED = ("drr_render", "drr_render_adjoint", "drr_render_adjoint_ws",
            "drr_adjoint_workspace_bytes", "drr_render_adjoint_noalloc", "drr_render_pose_grad",
            "drr_render_alpha_adjoint", "drr_render_alpha_adjoint_ws", "drr_poisson_noise", "drr_poisson_noise_backward",
            "drr_render_siddon", "drr_render_siddon_adjoint", "drr_render_batched",
            "drr_render_adjoint_batched", "drr_adjoint_batched_workspace_bytes",
            "drr_render_pose_grad_batched", "drr_render_alpha_adjoint_batched",
            "drr_render_adjoint_batched_ws", "drr_render_staged",
            "drr_prepared_bytes", "drr_prepare_volume", "drr_get_last_error", "drr_abi_version",
            "drr_wait_timeouts")
DRR_NOALLOC_SCRATCH_BYTES = 32 << 20


class DrrError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"libdrr status {status}: {message}")
        self.status = status


_lib = None
_c = ctypes
_vp = ctypes.c_void_p
_i3 = ctypes.c_int * 3
_f3 = ctypes.c_float * 3
_f9 = ctypes.c_float * 9


def use_library(path):
    """Load ``path`` (for example CHECKED_LIB_PATH, the bounds-checked debug
    build) in place of libdrr.so for every later call; returns the path that
    was in use, so that a caller can switch back."""
    global _lib, LIB_PATH
    previous = LIB_PATH
    LIB_PATH = path
    _lib = None
    return previous


def lib():
    """The loaded libdrr.so (built in-tree by cone_beam_ct_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libdrr.so is not built ({LIB_PATH}); run "
                           "`python -m cone_beam_ct_b200.build` -- there is no CPU fallback")
    L = ctypes.CDLL(LIB_PATH)
    L.drr_render.argtypes = [_vp, _c.c_int, _c.c_int, _i3, _f3, _f3, _f9, _vp, _c.c_int,
                             _c.c_int, _c.c_int, _c.c_int, _c.c_float, _c.c_int, _vp, _vp]
    L.drr_render.restype = _c.c_int
    L.drr_render_staged.argtypes = [_vp, _c.c_int, _i3, _f3, _f3, _f9, _vp, _c.c_int, _c.c_int,
                                    _c.c_int, _c.c_int, _c.c_float, _c.c_int, _vp, _vp]
    L.drr_render_staged.restype = _c.c_int
    L.drr_render_adjoint.argtypes = [_i3, _f3, _f3, _f9, _vp, _c.c_int, _c.c_int, _c.c_int,
                                     _c.c_int, _c.c_float, _c.c_int, _vp, _vp, _vp, _vp]
    L.drr_render_adjoint.restype = _c.c_int
    L.drr_render_adjoint_ws.argtypes = [_i3, _f3, _f3, _f9, _vp, _c.c_int, _c.c_int, _c.c_int,
                                        _c.c_int, _c.c_float, _c.c_int, _vp, _vp, _vp, _vp,
                                        _c.c_size_t, _vp]
    L.drr_render_adjoint_ws.restype = _c.c_int
    L.drr_render_adjoint_noalloc.argtypes = [_i3, _f3, _f3, _f9, _vp, _c.c_int, _c.c_int,
                                             _c.c_int, _c.c_int, _c.c_float, _c.c_int, _vp, _vp,
                                             _vp, _vp]
    L.drr_render_adjoint_noalloc.restype = _c.c_int
    L.drr_render_pose_grad.argtypes = [_vp, _c.c_int, _c.c_int, _i3, _f3, _f3, _f9, _vp,
                                       _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_float,
                                       _c.c_int, _vp, _vp, _vp, _vp]
    L.drr_render_pose_grad.restype = _c.c_int
    L.drr_render_pose_grad_batched.argtypes = [_vp, _c.c_int, _c.c_int, _i3, _f3, _f3, _f9, _vp,
                                               _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_int,
                                               _c.c_int, _c.c_float, _c.c_int, _vp, _vp, _vp,
                                               _vp]
    L.drr_render_pose_grad_batched.restype = _c.c_int
    L.drr_render_alpha_adjoint.argtypes = [_vp, _c.c_int, _c.c_int, _i3, _f3, _f3, _f9, _vp,
                                           _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_float,
                                           _vp, _vp, _vp, _vp]
    L.drr_render_alpha_adjoint.restype = _c.c_int
    L.drr_render_alpha_adjoint_ws.argtypes = [_vp, _c.c_int, _c.c_int, _i3, _f3, _f3, _f9, _vp,
                                              _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_float,
                                              _vp, _vp, _vp, _vp, _c.c_size_t, _vp]
    L.drr_render_alpha_adjoint_ws.restype = _c.c_int
    L.drr_render_alpha_adjoint_batched.argtypes = [_vp, _c.c_int, _c.c_int, _i3, _f3, _f3, _f9,
                                                   _vp, _c.c_int, _c.c_int, _c.c_int, _c.c_int,
                                                   _c.c_int, _c.c_int, _c.c_float, _vp, _vp, _vp,
                                                   _vp, _c.c_size_t, _vp]
    L.drr_render_alpha_adjoint_batched.restype = _c.c_int
    L.drr_poisson_noise.argtypes = [_vp, _vp, _c.c_float, _vp, _c.c_int64, _vp]
    L.drr_poisson_noise.restype = _c.c_int
    L.drr_poisson_noise_backward.argtypes = [_vp, _vp, _c.c_float, _vp, _vp, _c.c_int64, _vp]
    L.drr_poisson_noise_backward.restype = _c.c_int
    L.drr_render_siddon.argtypes = [_vp, _c.c_int, _i3, _f3, _f3, _f9, _vp, _c.c_int, _c.c_int,
                                    _c.c_int, _c.c_float, _c.c_int, _vp, _vp]
    L.drr_render_siddon.restype = _c.c_int
    L.drr_render_siddon_adjoint.argtypes = [_i3, _f3, _f3, _f9, _vp, _c.c_int, _c.c_int,
                                            _c.c_int, _c.c_float, _c.c_int, _vp, _vp, _vp, _vp]
    L.drr_render_siddon_adjoint.restype = _c.c_int
    L.drr_render_batched.argtypes = [_vp, _c.c_int, _c.c_int, _i3, _f3, _f3, _f9, _vp,
                                     _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_int,
                                     _c.c_float, _c.c_int, _vp, _vp]
    L.drr_render_batched.restype = _c.c_int
    L.drr_render_adjoint_batched.argtypes = [_i3, _f3, _f3, _f9, _vp, _c.c_int, _c.c_int,
                                             _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_float,
                                             _c.c_int, _vp, _vp, _vp, _vp]
    L.drr_render_adjoint_batched.restype = _c.c_int
    L.drr_adjoint_workspace_bytes.argtypes = [_i3, _c.c_int]
    L.drr_adjoint_workspace_bytes.restype = _c.c_size_t
    L.drr_adjoint_batched_workspace_bytes.argtypes = [_i3, _c.c_int, _c.c_int, _c.c_int]
    L.drr_adjoint_batched_workspace_bytes.restype = _c.c_size_t
    L.drr_render_adjoint_batched_ws.argtypes = (L.drr_render_adjoint_batched.argtypes[:-1] +
                                                [_vp, _c.c_size_t, _vp])
    L.drr_render_adjoint_batched_ws.restype = _c.c_int
    L.drr_prepared_bytes.argtypes = [_i3, _c.c_int, _c.c_int]
    L.drr_prepared_bytes.restype = _c.c_size_t
    L.drr_prepare_volume.argtypes = [_vp, _i3, _c.c_int, _c.c_int, _vp, _c.c_size_t, _vp]
    L.drr_prepare_volume.restype = _c.c_int
    L.drr_get_last_error.argtypes = []
    L.drr_get_last_error.restype = _c.c_char_p
    L.drr_abi_version.argtypes = []
    L.drr_abi_version.restype = _c.c_int
    L.drr_wait_timeouts.argtypes = [_c.POINTER(_c.c_ulonglong)]
    L.drr_wait_timeouts.restype = _c.c_int
    if hasattr(L, "drr_debug_bounds_errors"):
        L.drr_debug_bounds_errors.argtypes = [_c.POINTER(_c.c_ulonglong), _c.POINTER(_c.c_longlong)]
        L.drr_debug_bounds_errors.restype = _c.c_int
    _lib = L
    return L


def _dev(x, name, allow_none=False):
    """Device address of a CUDA tensor (or an int address)."""
    if x is None:
        if allow_none:
            return None
        raise TypeError(f"{name} must be a CUDA tensor or a device address")
    if isinstance(x, int):
        return x
    if not getattr(x, "is_cuda", False):
        raise TypeError(f"{name} must live on a CUDA device")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _i3v(v):
    a = np.asarray(v, dtype=np.int64).reshape(-1)
    if a.size != 3:
        raise ValueError("expected 3 values")
    return _i3(*(int(x) for x in a))


def _f3v(v):
    a = np.asarray(v, dtype=np.float32).reshape(-1)
    if a.size != 3:
        raise ValueError("expected 3 values")
    return _f3(*(float(x) for x in a))


def _f9v(v):
    a = np.asarray(v, dtype=np.float32).reshape(-1)
    if a.size != 9:
        raise ValueError("K must have 9 values")
    return _f9(*(float(x) for x in a))


def _check(status):
    if status != DRR_OK:
        raise DrrError(status, drr_get_last_error())


def drr_get_last_error():
    return lib().drr_get_last_error().decode()


def drr_abi_version():
    return lib().drr_abi_version()


def drr_prepared_bytes(dims, dtype, layout):
    return int(lib().drr_prepared_bytes(_i3v(dims), int(dtype), int(layout)))


def drr_prepare_volume(src, dims, dtype, layout, dst, dst_bytes=None, stream=None):
    if dst_bytes is None:
        dst_bytes = dst.numel() * dst.element_size()
    _check(lib().drr_prepare_volume(_dev(src, "src"), _i3v(dims), int(dtype), int(layout),
                                    _dev(dst, "dst"), int(dst_bytes), _stream(stream)))


def drr_render(vol, dtype, layout, dims, spacing, origin, K, Rt, B, H, W, n_samples,
               density_factor, mode, out, stream=None):
    _check(lib().drr_render(_dev(vol, "vol", True), int(dtype), int(layout), _i3v(dims),
                            _f3v(spacing), _f3v(origin), _f9v(K), _dev(Rt, "Rt", True), int(B),
                            int(H), int(W), int(n_samples), float(density_factor), int(mode),
                            _dev(out, "out", True), _stream(stream)))


def drr_render_staged(vol, dtype, dims, spacing, origin, K, Rt, B, H, W, n_samples,
                      density_factor, mode, out, stream=None):
    _check(lib().drr_render_staged(_dev(vol, "vol", True), int(dtype), _i3v(dims), _f3v(spacing),
                                   _f3v(origin), _f9v(K), _dev(Rt, "Rt", True), int(B), int(H),
                                   int(W), int(n_samples), float(density_factor), int(mode),
                                   _dev(out, "out", True), _stream(stream)))


def drr_render_adjoint(dims, spacing, origin, K, Rt, B, H, W, n_samples, density_factor, mode,
                       grad_out, fwd_out, grad_vol, stream=None):
    _check(lib().drr_render_adjoint(_i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                    _dev(Rt, "Rt", True), int(B), int(H), int(W), int(n_samples),
                                    float(density_factor), int(mode),
                                    _dev(grad_out, "grad_out", True),
                                    _dev(fwd_out, "fwd_out", True),
                                    _dev(grad_vol, "grad_vol", True), _stream(stream)))


def drr_render_pose_grad(vol, dtype, layout, dims, spacing, origin, K, Rt, B, H, W, n_samples,
                         density_factor, mode, grad_out, fwd_out, grad_Rt, stream=None):
    _check(lib().drr_render_pose_grad(_dev(vol, "vol", True), int(dtype), int(layout), _i3v(dims),
                                      _f3v(spacing), _f3v(origin), _f9v(K), _dev(Rt, "Rt", True),
                                      int(B), int(H), int(W), int(n_samples),
                                      float(density_factor), int(mode),
                                      _dev(grad_out, "grad_out", True),
                                      _dev(fwd_out, "fwd_out", True),
                                      _dev(grad_Rt, "grad_Rt", True), _stream(stream)))


def drr_render_pose_grad_batched(vols, dtype, layout, dims, spacing, origin, K, Rt, n_vols,
                                 channels, n_views, H, W, n_samples, density_factor, mode,
                                 grad_out, fwd_out, grad_Rt, stream=None):
    _check(lib().drr_render_pose_grad_batched(_dev(vols, "vols", True), int(dtype), int(layout),
                                              _i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                              _dev(Rt, "Rt", True), int(n_vols), int(channels),
                                              int(n_views), int(H), int(W), int(n_samples),
                                              float(density_factor), int(mode),
                                              _dev(grad_out, "grad_out", True),
                                              _dev(fwd_out, "fwd_out", True),
                                              _dev(grad_Rt, "grad_Rt", True), _stream(stream)))


def drr_render_alpha_adjoint(vol, dtype, layout, dims, spacing, origin, K, Rt, B, H, W,
                             n_samples, density_factor, grad_out, fwd_out, grad_vol, stream=None):
    _check(lib().drr_render_alpha_adjoint(_dev(vol, "vol", True), int(dtype), int(layout),
                                          _i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                          _dev(Rt, "Rt", True), int(B), int(H), int(W),
                                          int(n_samples), float(density_factor),
                                          _dev(grad_out, "grad_out", True),
                                          _dev(fwd_out, "fwd_out", True),
                                          _dev(grad_vol, "grad_vol", True), _stream(stream)))


def drr_render_alpha_adjoint_ws(vol, dtype, layout, dims, spacing, origin, K, Rt, B, H, W,
                                n_samples, density_factor, grad_out, fwd_out, grad_vol, workspace,
                                workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().drr_render_alpha_adjoint_ws(_dev(vol, "vol", True), int(dtype), int(layout),
                                             _i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                             _dev(Rt, "Rt", True), int(B), int(H), int(W),
                                             int(n_samples), float(density_factor),
                                             _dev(grad_out, "grad_out", True),
                                             _dev(fwd_out, "fwd_out", True),
                                             _dev(grad_vol, "grad_vol", True),
                                             _dev(workspace, "workspace", True),
                                             int(workspace_bytes), _stream(stream)))


def drr_render_alpha_adjoint_batched(vols, dtype, layout, dims, spacing, origin, K, Rt, n_vols,
                                     channels, n_views, H, W, n_samples, density_factor,
                                     grad_out, fwd_out, grad_vols, workspace=None,
                                     workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().drr_render_alpha_adjoint_batched(_dev(vols, "vols", True), int(dtype),
                                                  int(layout), _i3v(dims), _f3v(spacing),
                                                  _f3v(origin), _f9v(K), _dev(Rt, "Rt", True),
                                                  int(n_vols), int(channels), int(n_views),
                                                  int(H), int(W), int(n_samples),
                                                  float(density_factor),
                                                  _dev(grad_out, "grad_out", True),
                                                  _dev(fwd_out, "fwd_out", True),
                                                  _dev(grad_vols, "grad_vols", True),
                                                  _dev(workspace, "workspace", True),
                                                  int(workspace_bytes), _stream(stream)))


def drr_poisson_noise(image, z, i0, out, n=None, stream=None):
    n = image.numel() if n is None else n
    _check(lib().drr_poisson_noise(_dev(image, "image", True), _dev(z, "z", True), float(i0),
                                   _dev(out, "out", True), int(n), _stream(stream)))


def drr_poisson_noise_backward(image, z, i0, grad_out, grad_image, n=None, stream=None):
    n = image.numel() if n is None else n
    _check(lib().drr_poisson_noise_backward(_dev(image, "image", True), _dev(z, "z", True),
                                            float(i0), _dev(grad_out, "grad_out", True),
                                            _dev(grad_image, "grad_image", True), int(n),
                                            _stream(stream)))


def drr_render_siddon(vol, dtype, dims, spacing, origin, K, Rt, B, H, W, density_factor, mode,
                      out, stream=None):
    _check(lib().drr_render_siddon(_dev(vol, "vol", True), int(dtype), _i3v(dims), _f3v(spacing),
                                   _f3v(origin), _f9v(K), _dev(Rt, "Rt", True), int(B), int(H),
                                   int(W), float(density_factor), int(mode),
                                   _dev(out, "out", True), _stream(stream)))


def drr_render_siddon_adjoint(dims, spacing, origin, K, Rt, B, H, W, density_factor, mode,
                              grad_out, fwd_out, grad_vol, stream=None):
    _check(lib().drr_render_siddon_adjoint(_i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                           _dev(Rt, "Rt", True), int(B), int(H), int(W),
                                           float(density_factor), int(mode),
                                           _dev(grad_out, "grad_out", True),
                                           _dev(fwd_out, "fwd_out", True),
                                           _dev(grad_vol, "grad_vol", True), _stream(stream)))


def drr_render_batched(vols, dtype, layout, dims, spacing, origin, K, Rt, n_vols, channels,
                       n_views, H, W, n_samples, density_factor, mode, out, stream=None):
    _check(lib().drr_render_batched(_dev(vols, "vols", True), int(dtype), int(layout), _i3v(dims),
                                    _f3v(spacing), _f3v(origin), _f9v(K), _dev(Rt, "Rt", True),
                                    int(n_vols), int(channels), int(n_views), int(H), int(W),
                                    int(n_samples), float(density_factor), int(mode),
                                    _dev(out, "out", True), _stream(stream)))


def drr_render_adjoint_batched(dims, spacing, origin, K, Rt, n_vols, channels, n_views, H, W,
                               n_samples, density_factor, mode, grad_out, fwd_out, grad_vols,
                               stream=None):
    _check(lib().drr_render_adjoint_batched(_i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                            _dev(Rt, "Rt", True), int(n_vols), int(channels),
                                            int(n_views), int(H), int(W), int(n_samples),
                                            float(density_factor), int(mode),
                                            _dev(grad_out, "grad_out", True),
                                            _dev(fwd_out, "fwd_out", True),
                                            _dev(grad_vols, "grad_vols", True), _stream(stream)))


def drr_adjoint_workspace_bytes(dims, B):
    return int(lib().drr_adjoint_workspace_bytes(_i3v(dims), int(B)))


def drr_adjoint_batched_workspace_bytes(dims, n_vols, channels, n_views):
    return int(lib().drr_adjoint_batched_workspace_bytes(_i3v(dims), int(n_vols), int(channels),
                                                         int(n_views)))


def drr_render_adjoint_batched_ws(dims, spacing, origin, K, Rt, n_vols, channels, n_views, H, W,
                                  n_samples, density_factor, mode, grad_out, fwd_out, grad_vols,
                                  workspace, workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().drr_render_adjoint_batched_ws(_i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                               _dev(Rt, "Rt", True), int(n_vols), int(channels),
                                               int(n_views), int(H), int(W), int(n_samples),
                                               float(density_factor), int(mode),
                                               _dev(grad_out, "grad_out", True),
                                               _dev(fwd_out, "fwd_out", True),
                                               _dev(grad_vols, "grad_vols", True),
                                               _dev(workspace, "workspace", True),
                                               int(workspace_bytes), _stream(stream)))


def drr_render_adjoint_ws(dims, spacing, origin, K, Rt, B, H, W, n_samples, density_factor, mode,
                          grad_out, fwd_out, grad_vol, workspace, workspace_bytes=None,
                          stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().drr_render_adjoint_ws(_i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                       _dev(Rt, "Rt", True), int(B), int(H), int(W),
                                       int(n_samples), float(density_factor), int(mode),
                                       _dev(grad_out, "grad_out", True),
                                       _dev(fwd_out, "fwd_out", True),
                                       _dev(grad_vol, "grad_vol", True),
                                       _dev(workspace, "workspace", True), int(workspace_bytes),
                                       _stream(stream)))


def drr_render_adjoint_noalloc(dims, spacing, origin, K, Rt, B, H, W, n_samples, density_factor,
                               mode, grad_out, fwd_out, grad_vol, stream=None):
    """drr_render_adjoint for callers that may not allocate device memory:
    the library's built-in 32 MiB scratch serves as the workspace."""
    _check(lib().drr_render_adjoint_noalloc(_i3v(dims), _f3v(spacing), _f3v(origin), _f9v(K),
                                            _dev(Rt, "Rt", True), int(B), int(H), int(W),
                                            int(n_samples), float(density_factor), int(mode),
                                            _dev(grad_out, "grad_out", True),
                                            _dev(fwd_out, "fwd_out", True),
                                            _dev(grad_vol, "grad_vol", True), _stream(stream)))


def drr_wait_timeouts():
    """Grid-barrier waits of the adjoint's slab pass that gave up on the
    current device since the last call (0 in normal operation); the count is
    cleared.  Call after the work has completed."""
    count = _c.c_ulonglong(0)
    _check(lib().drr_wait_timeouts(_c.byref(count)))
    return int(count.value)


def drr_debug_bounds_errors():
    """(count, first offset) of out-of-range accesses since the last call, from
    the bounds-checked build (use_library(CHECKED_LIB_PATH)); the device
    words are cleared.  Call after the work has completed."""
    L = lib()
    if not hasattr(L, "drr_debug_bounds_errors"):
        raise RuntimeError(f"{LIB_PATH} is not the bounds-checked build")
    count, first = _c.c_ulonglong(0), _c.c_longlong(0)
    _check(L.drr_debug_bounds_errors(_c.byref(count), _c.byref(first)))
    return int(count.value), int(first.value)

"""Texture-trilinear comparison (libdrr_texture.so), measured against the
oracle.  The texture units weight the 8 corners with 8-bit fixed-point
fractions (TorchTomo page, "Fast CUDA Kernels": ~1e-4 relative from the
exact forward), so the path is accepted only where it meets the parity
tolerance (1e-4 for fp32 volumes, 1e-2 for bf16-class storage).  These tests
measure and record the errors; they pin the decision, not a pass for the
texture path."""
import json
import os

import numpy as np
import pytest

import oracle
from cone_beam_ct_b200 import workloads as wl
from tests.gpu_helpers import parity_errors

pytestmark = pytest.mark.gpu
TOL_F32, TOL_BF16 = 1e-4, 1e-2


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from cone_beam_ct_b200 import texture
    texture.lib()
    return torch


def texture_forward(w, texel, Rt=None):
    import torch
    from cone_beam_ct_b200 import texture
    v = torch.from_numpy(w.vol).cuda()
    Rt_d = torch.from_numpy(np.ascontiguousarray((w.Rt if Rt is None else Rt).reshape(-1, 12))).cuda()
    B = Rt_d.shape[0]
    out = torch.empty((B, w.H, w.W), dtype=torch.float32, device="cuda")
    tv = texture.TextureVolume(v, w.dims, texel)
    try:
        tv.render(w.spacing, w.origin, w.K, Rt_d, B, w.H, w.W, w.n_samples, w.density_factor,
                  w.mode, out)
        torch.cuda.synchronize()
    finally:
        tv.close()
    return out.cpu().numpy()


def _record(name, texel, norm, rel):
    """Append the measured errors to the file DRR_TEXTURE_ERRORS names, if set."""
    path = os.environ.get("DRR_TEXTURE_ERRORS")
    if not path:
        return
    with open(path, "a") as f:
        f.write(json.dumps({"case": name, "texel": texel, "normwise": norm, "per_pixel": rel}) + "\n")


@pytest.mark.parametrize("texel", [0, 1])
def test_texture_error_config1(cuda, texel):
    w = wl.make_config(1)
    got = texture_forward(w, texel)
    ref = oracle.render(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                        w.density_factor, w.mode)
    norm, rel = parity_errors(got, ref)
    _record("config1", texel, norm, rel)
    assert norm < 5e-2, "texture path far off: a broken comparison, not just 8-bit weights"


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [2, 3])
@pytest.mark.parametrize("texel", [0, 1])
def test_texture_error_sampled(cuda, cfg, texel):
    w = wl.make_config(cfg)
    Rt = w.Rt[:2]
    got = texture_forward(w, texel, Rt=Rt)
    rng = np.random.default_rng(cfg)
    ids = rng.choice(2 * w.H * w.W, size=20000, replace=False)
    ref = oracle.render_rays(w.vol, w.dims, w.spacing, w.origin, w.K, Rt, w.H, w.W, w.n_samples,
                             w.density_factor, w.mode, ids)
    norm, rel = parity_errors(got.reshape(-1)[ids], ref)
    _record(f"config{cfg}", texel, norm, rel)
    assert norm < 5e-2

"""B200-native cone-beam DRR ray-marcher (forward projection and its adjoint).

The compute path is libdrr.so (hand-written sm_100a CUDA behind the C ABI of
include/drr.h): the forward ray-march, its volume adjoint and its pose
gradient; ``cone_beam_ct_b200.drr`` binds it with the same names.
``cone_beam_ct_b200.workloads`` makes seeded synthetic inputs.
"""
from .drr import (  # noqa: F401
    DRR_BF16,
    DRR_F32,
    DRR_LAYOUT_BRICKS,
    DRR_LAYOUT_CORNERS,
    DRR_LAYOUT_LINEAR,
    DRR_LAYOUT_PADDED,
    DRR_LAYOUT_QUADS,
    DRR_MODE_ALPHA,
    DRR_MODE_BEER_LAMBERT,
    DRR_MODE_RAW,
    DrrError,
    drr_abi_version,
    drr_adjoint_batched_workspace_bytes,
    drr_adjoint_workspace_bytes,
    drr_get_last_error,
    drr_poisson_noise,
    drr_poisson_noise_backward,
    drr_prepare_volume,
    drr_prepared_bytes,
    drr_render,
    drr_render_adjoint,
    drr_render_adjoint_batched,
    drr_render_adjoint_batched_ws,
    drr_render_alpha_adjoint,
    drr_render_alpha_adjoint_batched,
    drr_render_alpha_adjoint_ws,
    drr_render_batched,
    drr_render_adjoint_noalloc,
    drr_render_adjoint_ws,
    drr_render_pose_grad,
    drr_render_pose_grad_batched,
    drr_render_siddon,
    drr_render_siddon_adjoint,
    drr_render_staged,
    drr_wait_timeouts,
)

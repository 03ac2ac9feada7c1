"""fp64 CPU oracle of the cone-beam DRR ray-march -- TEST INFRASTRUCTURE.

Only tests/, the smoke check in __graft_entry__ and the cpu_baseline leg of
bench.py may import this package.  The product path (cone_beam_ct_b200)
never imports it and shares no code with it.
"""
from .oracle import (  # noqa: F401
    adjoint,
    adjoint_batched,
    batch_map,
    bf16_to_float,
    build,
    load,
    poisson_noise,
    poisson_noise_backward,
    pose_grad,
    pose_grad_batched,
    ray,
    render,
    render_batched,
    render_rays,
    render_siddon,
    round_bf16,
    siddon_adjoint,
    trilinear,
)

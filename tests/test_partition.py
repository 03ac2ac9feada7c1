"""The multi-GPU partition of one job (cone_beam_ct_b200.partition: detector
rows split over ranks, the volume replicated; diffct page, "Multi-GPU and
multi-node") on CPU: the split itself, the row-block intrinsics, and two
gloo ranks whose per-rank compute is the fp64 oracle, so that the partition,
the volume broadcast and the gradient all-reduce are checked against the
single-rank oracle result without a GPU."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
from cone_beam_ct_b200 import partition as P
from cone_beam_ct_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("B,H,world", [(4, 1024, 8), (4, 1024, 3), (1, 10, 4), (64, 200, 8),
                                       (2, 3, 5), (3, 7, 1)])
def test_shares_cover_every_row_once_in_order(B, H, world):
    W = 5
    seen = []
    sizes = []
    for rank in range(world):
        part = P.Partition(B, H, W, world, rank)
        assert len(part.segments) <= 3
        off = 0
        for s in part.segments:
            assert s.offset == off
            off += s.n_views * s.rows * W
            assert 0 <= s.row0 and s.row0 + s.rows <= H and s.view0 + s.n_views <= B
            seen += [v * H + r for v in range(s.view0, s.view0 + s.n_views)
                     for r in range(s.row0, s.row0 + s.rows)]
        assert off == part.rows * W
        sizes.append(part.rows)
    assert seen == list(range(B * H))
    assert max(sizes) - min(sizes) <= 1


def test_row_block_intrinsics_map_block_rows_to_detector_rows():
    # K^-1 (u, v, 1) of the block's row r equals K^-1 (u, r0 + r, 1) of the detector
    K = np.array([[2550.0, 0.3, 511.5], [0.0, 2549.0, 509.25], [0.0, 0.0, 1.25]])
    for r0 in (0, 1, 7, 512):
        Kb = P.row_block_K(K.reshape(-1).astype(np.float32), r0).astype(np.float64).reshape(3, 3)
        for u, r in ((0.0, 0.0), (100.0, 3.0), (1023.0, 17.0)):
            a = np.linalg.solve(Kb, [u, r, 1.0])
            b = np.linalg.solve(K.astype(np.float32).astype(np.float64), [u, r0 + r, 1.0])
            assert np.allclose(a, b, rtol=1e-12, atol=1e-15)


def _oracle_render(vol, dtype, layout, dims, spacing, origin, K, Rt, B, H, W, n_samples,
                   density_factor, mode, out, stream=None):
    img = oracle.render(vol.numpy(), dims, spacing, origin, np.asarray(K), Rt.numpy(), H, W,
                        n_samples, density_factor, mode)
    out.copy_(__import__("torch").from_numpy(img.reshape(-1)))


def _oracle_adjoint(vol):
    def adjoint(dims, spacing, origin, K, Rt, B, H, W, n_samples, density_factor, mode,
                grad_out, fwd_out, grad_vol, stream=None):
        import torch
        g = oracle.adjoint(dims, spacing, origin, np.asarray(K), Rt.numpy(), H, W, n_samples,
                           density_factor, mode, grad_out.numpy().reshape(B, H, W), vol=vol,
                           nthreads=1)
        grad_vol += torch.from_numpy(g)
    return adjoint


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    # 3 views of 23 rows: 2 ranks split view 1 in the middle of its rows
    return wl.small_random_case(41, B=3, H=23, W=19, n_samples=24)


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = _case()
        nx, ny, nz = w.dims
        vol = torch.from_numpy(w.vol.copy()) if rank == 0 else torch.zeros((nz, ny, nx))
        P.broadcast_volume(vol)
        part = P.Partition(w.B, w.H, w.W)
        assert (part.world, part.rank) == (world, rank)
        Rt = torch.from_numpy(np.ascontiguousarray(w.Rt.reshape(-1, 12)))
        out = torch.zeros(part.rays, dtype=torch.float64)
        P.render_partitioned(part, vol, 0, 0, w.dims, w.spacing, w.origin, w.K, Rt,
                             w.n_samples, w.density_factor, wl.MODE_RAW, out,
                             render=_oracle_render)
        # the whole image stack: each rank's rows in place, summed over ranks
        full = torch.zeros(w.B * w.H * w.W, dtype=torch.float64)
        full[part.local_slice()] = out
        dist.all_reduce(full)
        go = np.random.default_rng(9).standard_normal((w.B, w.H, w.W))
        go_local = torch.from_numpy(go.reshape(-1)[part.local_slice()].copy())
        grad = torch.zeros((nz, ny, nx), dtype=torch.float64)
        P.adjoint_partitioned(part, w.dims, w.spacing, w.origin, w.K, Rt, w.n_samples,
                              w.density_factor, wl.MODE_RAW, go_local, None, grad,
                              adjoint=_oracle_adjoint(vol.numpy()))
        q.put((rank, full.numpy(), grad.numpy(), float(vol.sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_single_rank_oracle():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict((r, rest) for r, *rest in (q.get(timeout=300) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = _case()
    img = oracle.render(w.vol, w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                        w.density_factor, wl.MODE_RAW).reshape(-1)
    go = np.random.default_rng(9).standard_normal((w.B, w.H, w.W))
    grad = oracle.adjoint(w.dims, w.spacing, w.origin, w.K, w.Rt, w.H, w.W, w.n_samples,
                          w.density_factor, wl.MODE_RAW, go, vol=w.vol, nthreads=1)
    for r in range(world):
        full, g, vsum = results[r]
        assert vsum == pytest.approx(float(w.vol.astype(np.float64).sum()), rel=1e-6)
        assert np.allclose(full, img, rtol=1e-12, atol=1e-12 * np.abs(img).max())
        # every rank holds the whole job's gradient after the all-reduce
        assert np.allclose(g, grad, rtol=1e-10, atol=1e-12 * np.abs(grad).max())

"""The bounded grid barrier that separates the phases of the volume
adjoint's slab pass (drr_barrier.cuh), driven by the probe library's
self-test: barriers that complete, and a barrier no epoch of which can
complete (one arrival more than the grid's CTAs) whose first wait runs out
after a short limit, makes every CTA return, and leaves the context usable.
No fault and no endless wait: the limit is a fraction of a second."""
import ctypes
import os
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROBE_LIB = os.path.join(ROOT, "cone_beam_ct_b200", "libdrr_probe.so")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def barrier():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()
    lib = ctypes.CDLL(PROBE_LIB)
    f = lib.drr_probe_grid_barrier
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p]
    f.restype = ctypes.c_int

    def run(extra, rounds, timeout_ms):
        t, p, c = ctypes.c_ulonglong(), ctypes.c_int(), ctypes.c_int()
        t0 = time.perf_counter()
        rc = f(extra, rounds, timeout_ms, ctypes.byref(t), ctypes.byref(p), ctypes.byref(c))
        assert rc == 0, f"drr_probe_grid_barrier returned {rc}"
        return t.value, p.value, c.value, time.perf_counter() - t0
    return run


def test_barriers_complete(barrier):
    timeouts, passes, ctas, _ = barrier(0, 200, 2000.0)
    assert timeouts == 0
    assert passes == 200 * ctas


def test_a_wait_that_runs_out_ends_every_cta_and_the_context_stays_usable(barrier):
    timeouts, passes, ctas, secs = barrier(1, 5, 100.0)
    assert passes == 0                      # no epoch could complete
    assert 1 <= timeouts <= ctas            # the first waits to run out raise the abort
    assert secs < 5.0                       # every CTA left soon after the limit
    timeouts, passes, ctas, _ = barrier(0, 10, 2000.0)
    assert timeouts == 0 and passes == 10 * ctas

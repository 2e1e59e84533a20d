"""Failure detection on the GPU without a fault: every wait of the tensor-core
kernels is bounded, and a wait that runs out records SSA_ERR_TIMEOUT in the
device error word and lets the kernel return.  ssa_wait_probe makes one such
wait run out on purpose (a barrier that nothing completes, a 100 us limit); the
test reads the status, checks that reading clears it, and that the context is
still usable by the next real call."""
import numpy as np
import pytest

from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import inputs, ops

from .helpers import to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from block_top_sparse_b200 import build
    build.build()


def test_wait_that_runs_out_reports_timeout_and_the_context_survives():
    torch.cuda.synchronize()
    assert L.ssa_get_device_error() == L.SSA_OK
    L.ssa_wait_probe(100_000)
    assert L.ssa_get_device_error() == L.SSA_ERR_TIMEOUT
    assert L.ssa_get_device_error() == L.SSA_OK  # reading cleared it
    # the context is intact: a real call runs and reports no error
    g = inputs.generate(inputs.WORKLOADS["long"], H=1, T=256)
    K = to_device(g["K"], "bf16")
    dims = L.make_dims(1, 1, 256, 128, 128, 1)
    Kbar = ops.block_pool(dims, K)
    torch.cuda.synchronize()
    assert L.ssa_get_device_error() == L.SSA_OK
    ref = inputs.to_float64(g["K"], "bf16").reshape(2, 128, 128).mean(axis=1)
    np.testing.assert_allclose(Kbar.cpu().numpy().reshape(2, 128), ref, rtol=2e-6, atol=1e-7)


def test_wait_probe_rejects_limits_outside_its_range():
    for bad in (0, 10, 2_000_000_000):
        with pytest.raises(L.SSAError) as e:
            L.ssa_wait_probe(bad)
        assert e.value.status == L.SSA_ERR_INVALID_ARG

"""The allocation-free full attention backward (ssa_full_attn_bwd_noalloc).

Some callers cannot allocate device memory where they call the backward: a
host framework that owns all device memory through its own pool, or a
latency-critical path where cudaMalloc (which can synchronise the device) is
not allowed.  This entry point keeps its scratch in an array inside libssa
instead of taking a workspace.  The test calls it twice in a row through the C
ABI and compares each result with the workspace entry point's result, using the
tolerances of the other parity tests, then a third time adding into the second
call's gradients (the scratch keeps the previous call's contents, so this checks
that the call clears what must start at zero); it also checks the size limit.

Kept in its own file, collected last, so that a run stopping at the first
failure has already run every other test.
"""
import pytest

from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import inputs, ops

from .helpers import check_close, to_device, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from block_top_sparse_b200 import build
    build.build()


@pytest.mark.parametrize("wlname,over", [("train", dict(B=1, H=2, T=1088)), ("tiny", dict(T=512))])
def test_noalloc_matches_workspace_entry_point(wlname, over):
    g = inputs.generate(inputs.WORKLOADS[wlname], with_dO=True, **over)
    w = g["wl"]
    dims = L.make_dims(w.B, w.H, w.T, w.d, w.s, 1, dtype=w.dtype)
    Q, K, V, dO = (to_device(g[key], w.dtype) for key in ("Q", "K", "V", "dO"))
    O, lse, O_lo = ops.attn_fwd(dims, Q, K, V)
    ref = [to_np(x) for x in ops.attn_bwd(dims, Q, K, V, O, lse, dO, O_lo=O_lo)]
    bf16 = w.dtype == "bf16"
    for call in range(2):
        dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
        L.ssa_full_attn_bwd_noalloc(dims, Q, K, V, O, lse, dO, dQ, dK, dV, 0, O_lo=O_lo)
        torch.cuda.synchronize()
        for name, got, r in zip(("dQ", "dK", "dV"), (dQ, dK, dV), ref):
            check_close("noalloc call %d %s" % (call, name), to_np(got), r, bf16)
    # third call: accumulate into the second call's results -> twice the gradients
    L.ssa_full_attn_bwd_noalloc(dims, Q, K, V, O, lse, dO, dQ, dK, dV, 1, O_lo=O_lo)
    torch.cuda.synchronize()
    for name, got, r in zip(("dQ", "dK", "dV"), (dQ, dK, dV), ref):
        check_close("noalloc accumulate %s" % name, to_np(got), 2 * r, bf16)
    assert L.ssa_get_device_error() == L.SSA_OK


def test_noalloc_rejects_problems_beyond_the_scratch():
    need_per_row = 4 + 128 * 4
    rows = L.SSA_NOALLOC_SCRATCH_BYTES // need_per_row + 128
    T = (rows // 128 + 1) * 128
    dims = L.make_dims(1, 1, T, 128, 128, 1)
    p = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.SSAError) as e:
        L.ssa_full_attn_bwd_noalloc(dims, p, p, p, p, p, p, p, p, p, 0, O_lo=p)
    assert e.value.status == L.SSA_ERR_WORKSPACE

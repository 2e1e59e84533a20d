"""Backward with O and O_lo off an 8-byte boundary.

The backward's row reduction D = rowsum(dO * (O + O_lo)) reads O and O_lo
with 8-byte loads (four rows per warp) when both are 8-byte aligned, and with
2-byte loads otherwise; the other inputs of the tensor-core path go through
TMA and must be 16-byte aligned anyway.  Both reductions give the same D up to
the order of the fp32 additions, so the gradients agree to fp32 rounding: the
test runs the backward once with the forward's O and O_lo and once with copies
placed two bytes past an 8-byte boundary, for the full and the sparse stream.
"""
import numpy as np
import pytest

from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import inputs, ops

from .helpers import rel_l2, to_device, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from block_top_sparse_b200 import build
    build.build()


def _offset_copy(t):
    """A copy of t whose data starts 2 bytes past an 8-byte boundary."""
    buf = torch.empty(t.numel() + 4, dtype=t.dtype, device=t.device)
    out = buf[1:1 + t.numel()].view(t.shape)
    out.copy_(t)
    assert out.data_ptr() % 8 == 2
    return out


@pytest.mark.parametrize("sparse", [False, True])
def test_backward_with_unaligned_output_rows(sparse):
    g = inputs.generate(inputs.WORKLOADS["train"], B=1, H=2, T=1024, with_dO=True)
    w = g["wl"]
    k = 4
    dims = L.make_dims(w.B, w.H, w.T, w.d, w.s, k, dtype=w.dtype)
    Q, K, V, dO = (to_device(g[key], w.dtype) for key in ("Q", "K", "V", "dO"))
    idx = None
    if sparse:
        Kbar = ops.block_pool(dims, K)
        idx = torch.empty((w.B, w.H, w.T, k), dtype=torch.int32, device="cuda")
        L.ssa_block_select(dims, Q, Kbar, idx)
    O, lse, O_lo = ops.attn_fwd(dims, Q, K, V, idx=idx)
    ref = ops.attn_bwd(dims, Q, K, V, O, lse, dO, idx=idx, O_lo=O_lo, grad_fp32=True)
    got = ops.attn_bwd(dims, Q, K, V, _offset_copy(O), lse, dO, idx=idx, O_lo=_offset_copy(O_lo), grad_fp32=True)
    torch.cuda.synchronize()
    assert L.ssa_get_device_error() == L.SSA_OK
    for name, a, b in zip(("dQ", "dK", "dV"), got, ref):
        a, b = to_np(a).astype(np.float64), to_np(b).astype(np.float64)
        assert np.all(np.isfinite(a)), name
        assert rel_l2(a, b) <= 1e-5, (name, rel_l2(a, b))

"""Allocation helpers and the full SSA attention step on top of the C ABI.

torch provides device memory and the stream only; every step runs in libssa's
kernels through the ``_lib`` binding.

``SSAStep`` chains one pass of the hot path for one batch:
  forward : pool -> select -> full attention -> sparse attention -> alignment loss
  backward: alignment grads (the main stream also receives its upstream dO)
            -> full attention backward -> sparse attention backward, both
            accumulating into the shared dQ, dK, dV.
The main stream is the one whose output feeds the rest of the model (paper
section 5 and Appendix C: full or sparse, drawn with probability 1/2 per step);
the other stream only receives the alignment gradient.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import _lib as L

_TORCH_DT = {"bf16": torch.bfloat16, "fp32": torch.float32}


def _ws(dims: L.Dims, op: int, device) -> Optional[torch.Tensor]:
    n = L.ssa_workspace_size(dims, op)
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def block_pool(dims: L.Dims, K: torch.Tensor) -> torch.Tensor:
    Kbar = torch.empty((dims.B, dims.H, dims.T // dims.s, dims.d), dtype=torch.float32, device=K.device)
    L.ssa_block_pool(dims, K, Kbar)
    return Kbar


def block_select(dims: L.Dims, Q: torch.Tensor, Kbar: torch.Tensor) -> torch.Tensor:
    idx = torch.empty((dims.B, dims.H, dims.T, dims.k), dtype=torch.int32, device=Q.device)
    L.ssa_block_select(dims, Q, Kbar, idx)
    return idx


def attn_fwd(dims: L.Dims, Q, K, V, idx: Optional[torch.Tensor] = None):
    O = torch.empty_like(Q)
    lse = torch.empty((dims.B, dims.H, dims.T), dtype=torch.float32, device=Q.device)
    if idx is None:
        L.ssa_full_attn_fwd(dims, Q, K, V, O, lse, _ws(dims, L.SSA_OP_FULL_FWD, Q.device))
    else:
        L.ssa_sparse_attn_fwd(dims, Q, K, V, idx, O, lse, _ws(dims, L.SSA_OP_SPARSE_FWD, Q.device))
    return O, lse


def attn_bwd(dims: L.Dims, Q, K, V, O, lse, dO, idx: Optional[torch.Tensor] = None, grads=None):
    """Returns (dQ, dK, dV); with ``grads`` given, adds into those tensors."""
    acc = grads is not None
    dQ, dK, dV = grads if acc else (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V))
    if idx is None:
        L.ssa_full_attn_bwd(dims, Q, K, V, O, lse, dO, dQ, dK, dV, int(acc), _ws(dims, L.SSA_OP_FULL_BWD, Q.device))
    else:
        L.ssa_sparse_attn_bwd(dims, Q, K, V, O, lse, dO, idx, dQ, dK, dV, int(acc),
                              _ws(dims, L.SSA_OP_SPARSE_BWD, Q.device))
    return dQ, dK, dV


def align_fwd(dims: L.Dims, Of, Os, beta=1.0, w_sparsity=1.0, w_commit=1.0) -> torch.Tensor:
    loss = torch.empty((), dtype=torch.float32, device=Of.device)
    L.ssa_align_loss_fwd(dims, Of, Os, beta, w_sparsity, w_commit, loss, _ws(dims, L.SSA_OP_ALIGN_FWD, Of.device))
    return loss


def align_bwd(dims: L.Dims, Of, Os, dloss, beta=1.0, w_sparsity=1.0, w_commit=1.0, dOf=None, dOs=None,
              accumulate=0):
    dOf = torch.empty_like(Of) if dOf is None else dOf
    dOs = torch.empty_like(Os) if dOs is None else dOs
    L.ssa_align_loss_bwd(dims, Of, Os, beta, w_sparsity, w_commit, dloss, dOf, dOs, accumulate)
    return dOf, dOs


def dropped_mass(dims: L.Dims, lse_sparse, lse_full) -> torch.Tensor:
    delta = torch.empty_like(lse_sparse)
    L.ssa_dropped_mass(dims, lse_sparse, lse_full, delta)
    return delta


class SSAStep:
    """Preallocated buffers for one pass of the hot path (forward + backward) at fixed dims."""

    def __init__(self, dims: L.Dims, device="cuda", main: str = "full", beta: float = 1.0,
                 w_sparsity: float = 1.0, w_commit: float = 1.0):
        assert main in ("full", "sparse")
        self.dims, self.main = dims, main
        self.beta, self.w_s, self.w_c = beta, w_sparsity, w_commit
        dt = torch.bfloat16 if dims.dtype == L.SSA_DT_BF16 else torch.float32
        B, H, T, d, s, k = dims.B, dims.H, dims.T, dims.d, dims.s, dims.k
        e = lambda *shape, dtype=dt: torch.empty(shape, dtype=dtype, device=device)  # noqa: E731
        self.Kbar = e(B, H, T // s, d, dtype=torch.float32)
        self.idx = e(B, H, T, k, dtype=torch.int32)
        self.Of, self.Os = e(B, H, T, d), e(B, H, T, d)
        self.lse_f, self.lse_s = e(B, H, T, dtype=torch.float32), e(B, H, T, dtype=torch.float32)
        self.loss = e(dtype=torch.float32)
        self.dloss = torch.ones((), dtype=torch.float32, device=device)
        self.dOf, self.dOs = e(B, H, T, d), e(B, H, T, d)
        self.dQ, self.dK, self.dV = e(B, H, T, d), e(B, H, T, d), e(B, H, T, d)
        self.ws: Dict[int, Optional[torch.Tensor]] = {
            op: _ws(dims, op, device) for op in (L.SSA_OP_SPARSE_FWD, L.SSA_OP_SPARSE_BWD, L.SSA_OP_FULL_FWD,
                                                 L.SSA_OP_FULL_BWD, L.SSA_OP_ALIGN_FWD)}

    # Number of libssa kernel launches per forward / backward (bf16, d = 128).
    KERNELS_FWD = 1 + 1 + 1 + (3 + 1 + 1) + 2      # pool, select, full, sparse(index x3, fwd, merge), align x2
    KERNELS_BWD = 1 + (1 + 1 + 1) + (3 + 1 + 1 + 1)  # align, full(prep, bwd, dq), sparse(index x3, prep, bwd, dq)

    def forward(self, Q, K, V, stream=None):
        d = self.dims
        L.ssa_block_pool(d, K, self.Kbar, stream)
        L.ssa_block_select(d, Q, self.Kbar, self.idx, L.SSA_SEL_FORCE_CURRENT, stream)
        L.ssa_full_attn_fwd(d, Q, K, V, self.Of, self.lse_f, self.ws[L.SSA_OP_FULL_FWD], stream)
        L.ssa_sparse_attn_fwd(d, Q, K, V, self.idx, self.Os, self.lse_s, self.ws[L.SSA_OP_SPARSE_FWD], stream)
        L.ssa_align_loss_fwd(d, self.Of, self.Os, self.beta, self.w_s, self.w_c, self.loss,
                             self.ws[L.SSA_OP_ALIGN_FWD], stream)
        return self.loss

    def backward(self, Q, K, V, stream=None):
        """Upstream gradient of the main stream must already sit in dOf (main='full') or dOs (main='sparse')."""
        d = self.dims
        acc = L.SSA_ACC_OF if self.main == "full" else L.SSA_ACC_OS
        L.ssa_align_loss_bwd(d, self.Of, self.Os, self.beta, self.w_s, self.w_c, self.dloss, self.dOf, self.dOs,
                             acc, stream)
        L.ssa_full_attn_bwd(d, Q, K, V, self.Of, self.lse_f, self.dOf, self.dQ, self.dK, self.dV, 0,
                            self.ws[L.SSA_OP_FULL_BWD], stream)
        L.ssa_sparse_attn_bwd(d, Q, K, V, self.Os, self.lse_s, self.dOs, self.idx, self.dQ, self.dK, self.dV, 1,
                              self.ws[L.SSA_OP_SPARSE_BWD], stream)
        return self.dQ, self.dK, self.dV

    def main_grad_buffer(self) -> torch.Tensor:
        return self.dOf if self.main == "full" else self.dOs

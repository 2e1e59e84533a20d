"""Allocation helpers and the full SSA attention step on top of the C ABI.

torch provides device memory and the stream only; every step runs in libssa's
kernels through the ``_lib`` binding.

``SSAStep`` chains one pass of the hot path for one batch:
  forward : pool -> select -> inverse index -> full attention -> sparse attention -> alignment loss
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
    Kbar = torch.empty((dims.B, dims.kv_heads, dims.T // dims.s, dims.d), dtype=torch.float32, device=K.device)
    L.ssa_block_pool(dims, K, Kbar)
    return Kbar


def block_select(dims: L.Dims, Q: torch.Tensor, Kbar: torch.Tensor) -> torch.Tensor:
    idx = torch.empty((dims.B, dims.kv_heads, dims.T, dims.k), dtype=torch.int32, device=Q.device)
    L.ssa_block_select(dims, Q, Kbar, idx)
    return idx


def sparse_index(dims: L.Dims, idx: torch.Tensor) -> Optional[torch.Tensor]:
    """Inverse selection index of idx (None for shapes whose kernels read idx directly)."""
    index = _ws(dims, L.SSA_OP_SPARSE_INDEX, idx.device)
    if index is not None:
        L.ssa_sparse_index(dims, idx, index)
    return index


def attn_fwd(dims: L.Dims, Q, K, V, idx: Optional[torch.Tensor] = None, index=None):
    """Returns (O, lse, O_lo): O_lo is the bf16 rounding residual of O (None for fp32)."""
    O = torch.empty_like(Q)
    O_lo = torch.empty_like(Q) if Q.dtype == torch.bfloat16 else None
    lse = torch.empty((dims.B, dims.H, dims.T), dtype=torch.float32, device=Q.device)
    if idx is None:
        L.ssa_full_attn_fwd(dims, Q, K, V, O, lse, _ws(dims, L.SSA_OP_FULL_FWD, Q.device), O_lo=O_lo)
    else:
        L.ssa_sparse_attn_fwd(dims, Q, K, V, idx, O, lse, _ws(dims, L.SSA_OP_SPARSE_FWD, Q.device), O_lo=O_lo,
                              index=index)
    return O, lse, O_lo


def attn_bwd(dims: L.Dims, Q, K, V, O, lse, dO, idx: Optional[torch.Tensor] = None, grads=None, O_lo=None,
             index=None, grad_fp32: bool = False):
    """Returns (dQ, dK, dV); with ``grads`` given, adds into those tensors.  grad_fp32: fp32 gradients."""
    acc = grads is not None
    gdt = torch.float32 if grad_fp32 else Q.dtype
    new = lambda t: torch.empty(t.shape, dtype=gdt, device=t.device)  # noqa: E731
    dQ, dK, dV = grads if acc else (new(Q), new(K), new(V))
    bits = (L.SSA_BWD_ACCUMULATE if acc else 0) | (L.SSA_BWD_GRAD_FP32 if grad_fp32 else 0)
    if idx is None:
        L.ssa_full_attn_bwd(dims, Q, K, V, O, lse, dO, dQ, dK, dV, bits, _ws(dims, L.SSA_OP_FULL_BWD, Q.device),
                            O_lo=O_lo)
    else:
        L.ssa_sparse_attn_bwd(dims, Q, K, V, O, lse, dO, idx, dQ, dK, dV, bits,
                              _ws(dims, L.SSA_OP_SPARSE_BWD, Q.device), O_lo=O_lo, index=index)
    return dQ, dK, dV


def align_fwd(dims: L.Dims, Of, Os, beta=1.0, w_sparsity=1.0, w_commit=1.0,
              kind=L.SSA_ALIGN_SMOOTH_L1) -> torch.Tensor:
    loss = torch.empty((), dtype=torch.float32, device=Of.device)
    L.ssa_align_loss_fwd(dims, Of, Os, beta, w_sparsity, w_commit, loss, _ws(dims, L.SSA_OP_ALIGN_FWD, Of.device),
                         kind=kind)
    return loss


def align_bwd(dims: L.Dims, Of, Os, dloss, beta=1.0, w_sparsity=1.0, w_commit=1.0, dOf=None, dOs=None,
              accumulate=0, kind=L.SSA_ALIGN_SMOOTH_L1):
    dOf = torch.empty_like(Of) if dOf is None else dOf
    dOs = torch.empty_like(Os) if dOs is None else dOs
    L.ssa_align_loss_bwd(dims, Of, Os, beta, w_sparsity, w_commit, dloss, dOf, dOs, accumulate, kind=kind)
    return dOf, dOs


def rope(dims: L.Dims, X: torch.Tensor, pos0: int = 0, base: float = 10000.0, factor: float = 1.0,
         transpose: bool = False) -> torch.Tensor:
    """Rotary position embedding of X [B, heads, T, d] in place (bf16 or fp32); returns X."""
    d = L.Dims(dims.B, dims.H, dims.T, dims.d, dims.s, dims.k,
               L.SSA_DT_FP32 if X.dtype == torch.float32 else L.SSA_DT_BF16, dims.scale, dims.Hkv)
    L.ssa_rope(d, X, X.shape[1], pos0, base, factor, int(transpose))
    return X


def dropped_mass(dims: L.Dims, lse_sparse, lse_full) -> torch.Tensor:
    delta = torch.empty_like(lse_sparse)
    L.ssa_dropped_mass(dims, lse_sparse, lse_full, delta)
    return delta


class SSAStep:
    """Preallocated buffers for one pass of the hot path (forward + backward) at fixed dims."""

    def __init__(self, dims: L.Dims, device="cuda", main: str = "full", beta: float = 1.0,
                 w_sparsity: float = 1.0, w_commit: float = 1.0, align_kind: int = L.SSA_ALIGN_SMOOTH_L1,
                 grad_fp32: bool = False, rope: Optional[tuple] = None):
        """grad_fp32: dQ, dK, dV in fp32, so the two streams' contributions are summed without rounding the
        first one to the input type.  rope = (base, factor): rotary positions are applied to copies of Q and K
        that the whole path reads, and dQ, dK are turned back to the unrotated inputs after the backward."""
        assert main in ("full", "sparse")
        self.grad_fp32 = grad_fp32
        self.rope = rope
        self.dims, self.main = dims, main
        self.beta, self.w_s, self.w_c, self.kind = beta, w_sparsity, w_commit, align_kind
        dt = torch.bfloat16 if dims.dtype == L.SSA_DT_BF16 else torch.float32
        B, H, T, d, s, k = dims.B, dims.H, dims.T, dims.d, dims.s, dims.k
        Hk = dims.kv_heads
        e = lambda *shape, dtype=dt: torch.empty(shape, dtype=dtype, device=device)  # noqa: E731
        self.Kbar = e(B, Hk, T // s, d, dtype=torch.float32)
        self.idx = e(B, Hk, T, k, dtype=torch.int32)
        self.Of, self.Os = e(B, H, T, d), e(B, H, T, d)
        # bf16 rounding residuals of the two outputs, read back by the backward passes
        self.Of_lo = e(B, H, T, d) if dt == torch.bfloat16 else None
        self.Os_lo = e(B, H, T, d) if dt == torch.bfloat16 else None
        self.index = _ws(dims, L.SSA_OP_SPARSE_INDEX, device)  # one inverse index per step
        self.Qr = e(B, H, T, d) if rope else None                # rotated copies of Q and K
        self.Kr = e(B, Hk, T, d) if rope else None
        self.lse_f, self.lse_s = e(B, H, T, dtype=torch.float32), e(B, H, T, dtype=torch.float32)
        self.loss = e(dtype=torch.float32)
        self.dloss = torch.ones((), dtype=torch.float32, device=device)
        self.dOf, self.dOs = e(B, H, T, d), e(B, H, T, d)
        gdt = torch.float32 if grad_fp32 else dt
        self.dQ, self.dK, self.dV = e(B, H, T, d, dtype=gdt), e(B, Hk, T, d, dtype=gdt), e(B, Hk, T, d, dtype=gdt)
        self.ws: Dict[int, Optional[torch.Tensor]] = {
            op: _ws(dims, op, device) for op in (L.SSA_OP_FULL_FWD, L.SSA_OP_FULL_BWD, L.SSA_OP_ALIGN_FWD)}
        # the sparse forward and backward share one workspace (they run one after the other on
        # the stream and keep nothing in it between calls)
        need = max(L.ssa_workspace_size(dims, L.SSA_OP_SPARSE_FWD), L.ssa_workspace_size(dims, L.SSA_OP_SPARSE_BWD))
        shared = torch.empty(need, dtype=torch.uint8, device=device) if need else None
        self.ws[L.SSA_OP_SPARSE_FWD] = self.ws[L.SSA_OP_SPARSE_BWD] = shared

    # Number of libssa kernel launches per forward (bf16, d = 128): pool, select, index (count, scan, fill,
    # launch order), full, sparse (kernel, merge), align (partial, final).
    KERNELS_FWD = 1 + 1 + 4 + 1 + (1 + 1) + 2

    def kernels_bwd(self) -> int:
        """libssa kernel launches per backward (bf16, d = 128): align, then per stream the prep and the
        attention kernel, plus the dQ conversion unless the gradients are fp32; with rotary positions the
        two passes that turn dQ and dK back."""
        per_stream = 2 if self.grad_fp32 else 3
        return 1 + 2 * per_stream + (2 if self.rope else 0)

    def _rotated(self, Q, K, stream=None):
        if not self.rope:
            return Q, K
        base, factor = self.rope
        self.Qr.copy_(Q)
        self.Kr.copy_(K)
        L.ssa_rope(self.dims, self.Qr, self.dims.H, 0, base, factor, 0, stream)
        L.ssa_rope(self.dims, self.Kr, self.dims.kv_heads, 0, base, factor, 0, stream)
        return self.Qr, self.Kr

    def forward(self, Q, K, V, stream=None):
        d = self.dims
        Q, K = self._rotated(Q, K, stream)
        L.ssa_block_pool(d, K, self.Kbar, stream)
        L.ssa_block_select(d, Q, self.Kbar, self.idx, L.SSA_SEL_FORCE_CURRENT, stream)
        if self.index is not None:
            L.ssa_sparse_index(d, self.idx, self.index, stream)
        L.ssa_full_attn_fwd(d, Q, K, V, self.Of, self.lse_f, self.ws[L.SSA_OP_FULL_FWD], stream, O_lo=self.Of_lo)
        L.ssa_sparse_attn_fwd(d, Q, K, V, self.idx, self.Os, self.lse_s, self.ws[L.SSA_OP_SPARSE_FWD], stream,
                              O_lo=self.Os_lo, index=self.index)
        L.ssa_align_loss_fwd(d, self.Of, self.Os, self.beta, self.w_s, self.w_c, self.loss,
                             self.ws[L.SSA_OP_ALIGN_FWD], stream, kind=self.kind)
        return self.loss

    def backward(self, Q, K, V, stream=None):
        """Upstream gradient of the main stream must already sit in dOf (main='full') or dOs (main='sparse')."""
        d = self.dims
        if self.rope:
            Q, K = self.Qr, self.Kr  # rotated by forward()
        acc = L.SSA_ACC_OF if self.main == "full" else L.SSA_ACC_OS
        L.ssa_align_loss_bwd(d, self.Of, self.Os, self.beta, self.w_s, self.w_c, self.dloss, self.dOf, self.dOs,
                             acc, stream, kind=self.kind)
        g32 = L.SSA_BWD_GRAD_FP32 if self.grad_fp32 else 0
        L.ssa_full_attn_bwd(d, Q, K, V, self.Of, self.lse_f, self.dOf, self.dQ, self.dK, self.dV, g32,
                            self.ws[L.SSA_OP_FULL_BWD], stream, O_lo=self.Of_lo)
        L.ssa_sparse_attn_bwd(d, Q, K, V, self.Os, self.lse_s, self.dOs, self.idx, self.dQ, self.dK, self.dV,
                              L.SSA_BWD_ACCUMULATE | g32, self.ws[L.SSA_OP_SPARSE_BWD], stream, O_lo=self.Os_lo,
                              index=self.index)
        if self.rope:
            base, factor = self.rope
            gd = L.Dims(d.B, d.H, d.T, d.d, d.s, d.k, L.SSA_DT_FP32 if self.grad_fp32 else d.dtype, d.scale, d.Hkv)
            L.ssa_rope(gd, self.dQ, d.H, 0, base, factor, 1, stream)
            L.ssa_rope(gd, self.dK, d.kv_heads, 0, base, factor, 1, stream)
        return self.dQ, self.dK, self.dV

    def main_grad_buffer(self) -> torch.Tensor:
        return self.dOf if self.main == "full" else self.dOs

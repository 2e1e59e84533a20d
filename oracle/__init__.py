"""fp64 CPU oracle for the SSA block-sparse attention path (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA path; the C source
``ssa_oracle.c`` is compiled with gcc/OpenMP into ``libssa_oracle.so`` beside it.

Functions take/return numpy arrays laid out [BH, T, d] (batch and heads
flattened) in float64, selections as int32 [BH, T, k].

What each function computes (readings of "SSA: Sparse Sparse Attention by
Aligning Full and Sparse Attention Outputs in Feature Space", paperlayer.ai
summary of v4):
  block_pool    section 3  mean-pooled block keys
  block_select  section 3  current block + top-(k-1) preceding blocks by q.Kbar
  block_scores  section 3  the candidate scores q.Kbar of chosen rows
  attn_fwd      sections 3 full causal attention / attention over the selected
                           blocks' tokens
  attn_bwd      section 4.2 gradients; dropped keys get none
  align_fwd/bwd section 5  bidirectional SmoothL1 output alignment; section 7.5
                           the adjusted L2 variant (kind="l2")
  dropped_mass  section 4.2 / Appendix B  delta = 1 - exp(lse_s - lse_f)
  rope          section 6 / Appendix K  rotary positions with a frequency scaling factor

Parity pins: see tests/test_oracle_pins.py.  Every function there is pinned
(brute force, library special cases, closed forms, invariants, finite
differences); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssa_oracle.c")
_LIB = os.path.join(_HERE, "libssa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle's C source (gcc -O2 -fopenmp); return the library path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    i64, dbl, p = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.ora_num_threads.restype = ctypes.c_int
    lib.ora_block_pool.argtypes = [i64, i64, i64, i64, p, p]
    lib.ora_block_select.argtypes = [i64, i64, i64, i64, i64, i64, p, p, p, p, p]
    lib.ora_block_scores.argtypes = [i64, i64, i64, i64, i64, i64, p, p, p, p, p]
    lib.ora_check_selection.argtypes = [i64, i64, i64, i64, p]
    lib.ora_check_selection.restype = ctypes.c_int
    lib.ora_attn_fwd.argtypes = [i64, i64, i64, i64, i64, i64, dbl, p, p, p, p, i64, p, p, p]
    lib.ora_attn_bwd.argtypes = [i64, i64, i64, i64, i64, i64, dbl, p, p, p, p, p, i64, p, i64, p, p, p, p,
                                 ctypes.c_int]
    lib.ora_rope.argtypes = [i64, i64, i64, p, i64, dbl, dbl, ctypes.c_int, p]
    lib.ora_align_fwd.argtypes = [i64, p, p, dbl, dbl, dbl, ctypes.c_int]
    lib.ora_align_fwd.restype = dbl
    lib.ora_align_bwd.argtypes = [i64, p, p, dbl, dbl, dbl, dbl, p, p, ctypes.c_int]
    _lib = lib
    return lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows) -> Optional[np.ndarray]:
    return None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)


def num_threads() -> int:
    return int(_load().ora_num_threads())


def block_pool(K: np.ndarray, s: int) -> np.ndarray:
    """K [BH, T, d] -> Kbar [BH, T/s, d]."""
    K = _f64(K)
    BH, T, d = K.shape
    out = np.empty((BH, T // s, d), dtype=np.float64)
    _load().ora_block_pool(BH, T, d, s, _ptr(K), _ptr(out))
    return out


def _group(nq: int, nk: int) -> int:
    """Query heads per key/value head (grouped-query attention); 1 when the counts agree."""
    if nk <= 0 or nq % nk:
        raise ValueError("query heads (%d) must be a multiple of key heads (%d)" % (nq, nk))
    return nq // nk


def block_select(Q: np.ndarray, Kbar: np.ndarray, s: int, k: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Q [BH, T, d], Kbar [BHk, nb, d] -> (idx int32 [BHk,T,k], r_(k-1) [BHk,T], r_(k) [BHk,T]).

    With BH = G * BHk (grouped query heads), key head g's selection scores block j by the sum over its G
    query heads of q . Kbar_j."""
    Q, Kbar = _f64(Q), _f64(Kbar)
    BH, T, d = Q.shape
    BHk = Kbar.shape[0]
    G = _group(BH, BHk)
    idx = np.empty((BHk, T, k), dtype=np.int32)
    r1 = np.empty((BHk, T), dtype=np.float64)
    r2 = np.empty((BHk, T), dtype=np.float64)
    _load().ora_block_select(BHk, G, T, d, s, k, _ptr(Q), _ptr(Kbar), _ptr(idx), _ptr(r1), _ptr(r2))
    return idx, r1, r2


def block_scores(Q: np.ndarray, Kbar: np.ndarray, s: int, bh, t) -> np.ndarray:
    """Candidate scores of the rows (key head bh[i], query t[i]) -> [n, nb] (NaN for j >= b(t))."""
    Q, Kbar = _f64(Q), _f64(Kbar)
    BH, T, d = Q.shape
    BHk = Kbar.shape[0]
    G = _group(BH, BHk)
    nb = T // s
    bh = np.ascontiguousarray(bh, dtype=np.int64)
    t = np.ascontiguousarray(t, dtype=np.int64)
    out = np.empty((bh.shape[0], nb), dtype=np.float64)
    _load().ora_block_scores(BHk, G, T, d, s, bh.shape[0], _ptr(bh), _ptr(t), _ptr(Q), _ptr(Kbar), _ptr(out))
    return out


def check_selection(idx: np.ndarray, s: int) -> bool:
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    BH, T, k = idx.shape
    return bool(_load().ora_check_selection(BH, T, s, k, _ptr(idx)))


def attn_fwd(Q, K, V, s: int, scale: float, idx: Optional[np.ndarray] = None, rows=None):
    """Full (idx None) or sparse attention forward -> (O [BH, n, d], lse [BH, n]).

    K, V (and idx) may have BH / G heads: query head bh then reads key head bh // G."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    BH, T, d = Q.shape
    G = _group(BH, K.shape[0])
    k = 0 if idx is None else idx.shape[-1]
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    rows = _rows(rows)
    n = T if rows is None else rows.shape[0]
    O = np.empty((BH, n, d), dtype=np.float64)
    lse = np.empty((BH, n), dtype=np.float64)
    _load().ora_attn_fwd(BH, G, T, d, s, k, float(scale), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                         n, _ptr(rows), _ptr(O), _ptr(lse))
    return O, lse


def attn_bwd(Q, K, V, dO, s: int, scale: float, idx: Optional[np.ndarray] = None, qrows=None, krows=None,
             stored_o: str = "exact"):
    """Gradients of sum(dO * O) -> (dQ [BH, nq, d], dK [BHk, nk, d], dV [BHk, nk, d]) (BHk = BH with one key
    head per query head; grouped query heads sum into their key head).

    stored_o="bf16": D_t = dO_t . o_t is formed with the oracle's own output rounded to bfloat16, the value
    a backward pass is given when the forward stores its output in bfloat16; "exact" uses o_t itself."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    BH, T, d = Q.shape
    G = _group(BH, K.shape[0])
    k = 0 if idx is None else idx.shape[-1]
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    qrows, krows = _rows(qrows), _rows(krows)
    nq = T if qrows is None else qrows.shape[0]
    nk = T if krows is None else krows.shape[0]
    dQ = np.empty((BH, nq, d), dtype=np.float64)
    dK = np.empty((BH // G, nk, d), dtype=np.float64)
    dV = np.empty((BH // G, nk, d), dtype=np.float64)
    _load().ora_attn_bwd(BH, G, T, d, s, k, float(scale), _ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(idx),
                         nq, _ptr(qrows), nk, _ptr(krows), _ptr(dQ), _ptr(dK), _ptr(dV),
                         1 if stored_o == "bf16" else 0)
    return dQ, dK, dV


def rope(X: np.ndarray, pos0: int = 0, base: float = 10000.0, factor: float = 1.0, inverse: bool = False):
    """Rotary position embedding of X [heads, T, d] (rotate-half pairs, angle (pos0+t) base^(-2i/d) / factor)."""
    X = _f64(X)
    heads, T, d = X.shape
    out = np.empty_like(X)
    _load().ora_rope(heads * T, T, d, _ptr(X), int(pos0), float(base), float(factor), 1 if inverse else 0,
                     _ptr(out))
    return out


ALIGN_KINDS = {"smooth_l1": 0, "l2": 1}


def align_fwd(Of, Os, beta: float = 1.0, w_sparsity: float = 1.0, w_commit: float = 1.0,
              kind: str = "smooth_l1") -> float:
    """Alignment loss; kind "smooth_l1" (section 5) or "l2" (the adjusted L2 variant of section 7.5)."""
    Of, Os = _f64(Of).ravel(), _f64(Os).ravel()
    return float(_load().ora_align_fwd(Of.size, _ptr(Of), _ptr(Os), beta, w_sparsity, w_commit, ALIGN_KINDS[kind]))


def align_bwd(Of, Os, beta: float = 1.0, w_sparsity: float = 1.0, w_commit: float = 1.0, g: float = 1.0,
              kind: str = "smooth_l1"):
    shape = np.shape(Of)
    Of, Os = _f64(Of).ravel(), _f64(Os).ravel()
    dOf = np.empty_like(Of)
    dOs = np.empty_like(Os)
    _load().ora_align_bwd(Of.size, _ptr(Of), _ptr(Os), beta, w_sparsity, w_commit, g, _ptr(dOf), _ptr(dOs),
                          ALIGN_KINDS[kind])
    return dOf.reshape(shape), dOs.reshape(shape)


def dropped_mass(lse_sparse: np.ndarray, lse_full: np.ndarray) -> np.ndarray:
    """Page section 4.2 / Appendix B: full-attention mass outside S(t), delta = 1 - exp(lse_s - lse_f)."""
    return 1.0 - np.exp(_f64(lse_sparse) - _f64(lse_full))

"""ctypes binding of libssa.so (include/ssa.h): argument marshalling only.

Each ``ssa_*`` function here has the name and argument order of the C entry
point.  Device buffers are passed as torch CUDA tensors (their data pointers
go to the library unchanged), the stream defaults to torch's current stream.
Every computation runs in the library's CUDA kernels; there is no fallback:
if libssa.so is missing or cannot be loaded, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssa.so")

(SSA_OK, SSA_ERR_INVALID_ARG, SSA_ERR_UNSUPPORTED, SSA_ERR_WORKSPACE, SSA_ERR_CUDA, SSA_ERR_TIMEOUT,
 SSA_ERR_BAD_INPUT) = range(7)
SSA_DT_BF16, SSA_DT_FP32 = 0, 1
(SSA_OP_SPARSE_FWD, SSA_OP_SPARSE_BWD, SSA_OP_FULL_FWD, SSA_OP_FULL_BWD, SSA_OP_ALIGN_FWD, SSA_OP_SPARSE_INDEX,
 SSA_OP_DECODE) = range(7)
SSA_SEL_FORCE_CURRENT = 1
SSA_ACC_OF, SSA_ACC_OS = 1, 2
SSA_ALIGN_SMOOTH_L1, SSA_ALIGN_L2 = 0, 1
SSA_BWD_ACCUMULATE, SSA_BWD_GRAD_FP32 = 1, 2
SSA_NOALLOC_SCRATCH_BYTES = 32 << 20

# Every entry point include/ssa.h declares.
EXPORTS = (
    "ssa_workspace_size", "ssa_block_pool", "ssa_block_select", "ssa_sparse_index", "ssa_sparse_attn_fwd",
    "ssa_sparse_attn_bwd",
    "ssa_full_attn_fwd", "ssa_full_attn_bwd", "ssa_align_loss_fwd", "ssa_align_loss_bwd", "ssa_dropped_mass",
    "ssa_get_device_error", "ssa_status_string", "ssa_full_attn_bwd_noalloc", "ssa_wait_probe",
    "ssa_sparse_decode", "ssa_rope",
)


class SSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s" % (fn, status_string(status)))


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32), ("d", ctypes.c_int32),
                ("s", ctypes.c_int32), ("k", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float),
                ("Hkv", ctypes.c_int32)]

    def __repr__(self):
        return "Dims(B=%d, H=%d, T=%d, d=%d, s=%d, k=%d, dtype=%d, scale=%g, Hkv=%d)" % (
            self.B, self.H, self.T, self.d, self.s, self.k, self.dtype, self.scale, self.Hkv)

    @property
    def kv_heads(self) -> int:
        return self.Hkv or self.H


def make_dims(B: int, H: int, T: int, d: int, s: int, k: int = 1, dtype: str = "bf16",
              scale: Optional[float] = None, Hkv: int = 0) -> Dims:
    """Hkv: key/value heads (0 = H); with Hkv < H the H query heads form groups of H / Hkv."""
    return Dims(B, H, T, d, s, k, SSA_DT_BF16 if dtype == "bf16" else SSA_DT_FP32,
                d ** -0.5 if scale is None else scale, Hkv)


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libssa.so (built in-tree by block_top_sparse_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libssa.so not found at %s; build it with `python -m block_top_sparse_b200.build`" % path)
    lib = ctypes.CDLL(path)
    P, C, I, U, F, S = ctypes.c_void_p, ctypes.POINTER(Dims), ctypes.c_int, ctypes.c_uint, ctypes.c_float, ctypes.c_size_t
    sig = {
        "ssa_workspace_size": (S, [C, I]),
        "ssa_block_pool": (I, [C, P, P, P]),
        "ssa_block_select": (I, [C, P, P, P, U, P]),
        "ssa_sparse_index": (I, [C, P, P, S, P]),
        "ssa_sparse_attn_fwd": (I, [C, P, P, P, P, P, P, P, P, P, S, P]),
        "ssa_sparse_attn_bwd": (I, [C, P, P, P, P, P, P, P, P, P, P, P, P, I, P, S, P]),
        "ssa_full_attn_fwd": (I, [C, P, P, P, P, P, P, P, S, P]),
        "ssa_full_attn_bwd": (I, [C, P, P, P, P, P, P, P, P, P, P, I, P, S, P]),
        "ssa_full_attn_bwd_noalloc": (I, [C, P, P, P, P, P, P, P, P, P, P, I, P]),
        "ssa_align_loss_fwd": (I, [C, P, P, I, F, F, F, P, P, S, P]),
        "ssa_align_loss_bwd": (I, [C, P, P, I, F, F, F, P, P, P, I, P]),
        "ssa_dropped_mass": (I, [C, P, P, P, P]),
        "ssa_get_device_error": (I, [P]),
        "ssa_wait_probe": (I, [ctypes.c_uint64, P]),
        "ssa_sparse_decode": (I, [C, P, P, P, P, P, P, P, P, P, S, P]),
        "ssa_rope": (I, [C, P, I, I, F, F, I, P]),
        "ssa_status_string": (ctypes.c_char_p, [I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().ssa_status_string(status).decode()


def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _check(fn: str, status: int) -> None:
    if status != SSA_OK:
        raise SSAError(fn, status)


def ssa_workspace_size(dims: Dims, op: int) -> int:
    return int(load().ssa_workspace_size(ctypes.byref(dims), op))


def ssa_block_pool(dims, K, Kbar, stream=None):
    _check("ssa_block_pool", load().ssa_block_pool(ctypes.byref(dims), _p(K), _p(Kbar), _stream(stream)))


def ssa_block_select(dims, Q, Kbar, idx, flags=SSA_SEL_FORCE_CURRENT, stream=None):
    _check("ssa_block_select",
           load().ssa_block_select(ctypes.byref(dims), _p(Q), _p(Kbar), _p(idx), flags, _stream(stream)))


def ssa_sparse_index(dims, idx, index, stream=None):
    _check("ssa_sparse_index",
           load().ssa_sparse_index(ctypes.byref(dims), _p(idx), _p(index), _nbytes(index), _stream(stream)))


def ssa_sparse_attn_fwd(dims, Q, K, V, idx, O, lse, ws=None, stream=None, O_lo=None, index=None):
    _check("ssa_sparse_attn_fwd",
           load().ssa_sparse_attn_fwd(ctypes.byref(dims), _p(Q), _p(K), _p(V), _p(idx), _p(index), _p(O), _p(O_lo),
                                      _p(lse), _p(ws), _nbytes(ws), _stream(stream)))


def ssa_sparse_attn_bwd(dims, Q, K, V, O, lse, dO, idx, dQ, dK, dV, accumulate=0, ws=None, stream=None, O_lo=None,
                        index=None):
    _check("ssa_sparse_attn_bwd",
           load().ssa_sparse_attn_bwd(ctypes.byref(dims), _p(Q), _p(K), _p(V), _p(O), _p(O_lo), _p(lse), _p(dO),
                                      _p(idx), _p(index), _p(dQ), _p(dK), _p(dV), int(accumulate), _p(ws),
                                      _nbytes(ws), _stream(stream)))


def ssa_full_attn_fwd(dims, Q, K, V, O, lse, ws=None, stream=None, O_lo=None):
    _check("ssa_full_attn_fwd",
           load().ssa_full_attn_fwd(ctypes.byref(dims), _p(Q), _p(K), _p(V), _p(O), _p(O_lo), _p(lse), _p(ws),
                                    _nbytes(ws), _stream(stream)))


def ssa_full_attn_bwd(dims, Q, K, V, O, lse, dO, dQ, dK, dV, accumulate=0, ws=None, stream=None, O_lo=None):
    _check("ssa_full_attn_bwd",
           load().ssa_full_attn_bwd(ctypes.byref(dims), _p(Q), _p(K), _p(V), _p(O), _p(O_lo), _p(lse), _p(dO),
                                    _p(dQ), _p(dK), _p(dV), int(accumulate), _p(ws), _nbytes(ws), _stream(stream)))


def ssa_full_attn_bwd_noalloc(dims, Q, K, V, O, lse, dO, dQ, dK, dV, accumulate=0, stream=None, O_lo=None):
    """Full attention backward with library-held scratch (no workspace, no allocation)."""
    _check("ssa_full_attn_bwd_noalloc",
           load().ssa_full_attn_bwd_noalloc(ctypes.byref(dims), _p(Q), _p(K), _p(V), _p(O), _p(O_lo), _p(lse),
                                            _p(dO), _p(dQ), _p(dK), _p(dV), int(accumulate), _stream(stream)))


def ssa_align_loss_fwd(dims, Of, Os, beta, w_sparsity, w_commit, loss, ws=None, stream=None,
                       kind=SSA_ALIGN_SMOOTH_L1):
    _check("ssa_align_loss_fwd",
           load().ssa_align_loss_fwd(ctypes.byref(dims), _p(Of), _p(Os), int(kind), beta, w_sparsity, w_commit,
                                     _p(loss), _p(ws), _nbytes(ws), _stream(stream)))


def ssa_align_loss_bwd(dims, Of, Os, beta, w_sparsity, w_commit, dloss, dOf, dOs, accumulate=0, stream=None,
                       kind=SSA_ALIGN_SMOOTH_L1):
    _check("ssa_align_loss_bwd",
           load().ssa_align_loss_bwd(ctypes.byref(dims), _p(Of), _p(Os), int(kind), beta, w_sparsity, w_commit,
                                     _p(dloss), _p(dOf), _p(dOs), int(accumulate), _stream(stream)))


def ssa_dropped_mass(dims, lse_sparse, lse_full, delta, stream=None):
    _check("ssa_dropped_mass",
           load().ssa_dropped_mass(ctypes.byref(dims), _p(lse_sparse), _p(lse_full), _p(delta), _stream(stream)))


def ssa_sparse_decode(dims, cache_len, q, Kcache, Vcache, Kbar_cache, idx, o, lse, ws=None, stream=None):
    _check("ssa_sparse_decode",
           load().ssa_sparse_decode(ctypes.byref(dims), _p(cache_len), _p(q), _p(Kcache), _p(Vcache), _p(Kbar_cache),
                                    _p(idx), _p(o), _p(lse), _p(ws), _nbytes(ws), _stream(stream)))


def ssa_rope(dims, X, heads, pos0=0, base=10000.0, factor=1.0, transpose=0, stream=None):
    _check("ssa_rope", load().ssa_rope(ctypes.byref(dims), _p(X), int(heads), int(pos0), base, factor, int(transpose),
                                       _stream(stream)))


def ssa_wait_probe(limit_ns: int, stream=None) -> None:
    _check("ssa_wait_probe", load().ssa_wait_probe(int(limit_ns), _stream(stream)))


def ssa_get_device_error(stream=None) -> int:
    return int(load().ssa_get_device_error(_stream(stream)))

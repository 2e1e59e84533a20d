"""Host-side checks of the C ABI: the library builds for sm_100a, loads, exports
every entry point include/ssa.h declares, and validates arguments on the host
(no kernel is launched: every call here fails validation before any CUDA call)."""
import ctypes
import os
import re

import pytest

from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ssa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ssa_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    assert names == sorted(L.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = os.popen("nm -D --defined-only %s" % L.LIB_PATH).read()
    for name in declared_functions():
        assert re.search(r"\bT %s\b" % name, out), name


def test_no_torch_in_boundary():
    src = open(os.path.join(ROOT, "include", "ssa.h")).read()
    assert "torch" not in src.lower() and "at::" not in src


def test_status_strings(lib):
    for code in range(7):
        assert L.status_string(code).startswith("SSA_")
    assert L.status_string(99) == "SSA_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    d = L.make_dims(1, 32, 32768, 128, 128, 16)
    # inverse index: entries and the list position of every (query, slot)
    ix = L.ssa_workspace_size(d, L.SSA_OP_SPARSE_INDEX)
    assert ix >= 32 * 32768 * 16 * (4 + 4)
    # sparse forward: index + fp16 partials + partial lse by list position
    sf = L.ssa_workspace_size(d, L.SSA_OP_SPARSE_FWD)
    assert sf >= ix + 32 * 32768 * 16 * (128 * 2 + 4)
    fb = L.ssa_workspace_size(d, L.SSA_OP_FULL_BWD)
    assert fb >= 32 * 32768 * (128 * 4 + 4)
    # sparse backward: D + index + the fp32 dQ accumulator
    sb = L.ssa_workspace_size(d, L.SSA_OP_SPARSE_BWD)
    assert sb >= fb + ix
    # shapes on the CUDA-core path read idx directly: no index
    assert L.ssa_workspace_size(L.make_dims(1, 2, 1024, 64, 64, 4, dtype="fp32"), L.SSA_OP_SPARSE_INDEX) == 0
    # grouped-query heads: the index is per key/value head, the partials per query head
    g = L.make_dims(1, 32, 32768, 128, 128, 16, Hkv=8)
    assert L.ssa_workspace_size(g, L.SSA_OP_SPARSE_INDEX) * 4 == pytest.approx(ix, rel=0.01)
    assert L.ssa_workspace_size(g, L.SSA_OP_SPARSE_FWD) == pytest.approx(sf - 3 * ix / 4, rel=0.01)
    assert L.ssa_workspace_size(d, L.SSA_OP_FULL_FWD) == 0
    assert L.ssa_workspace_size(d, L.SSA_OP_ALIGN_FWD) > 0
    # invalid dims -> 0
    assert L.ssa_workspace_size(L.make_dims(1, 1, 100, 128, 64, 1), L.SSA_OP_FULL_BWD) == 0
    # fp32 backward keeps three fp32 accumulators
    d32 = L.make_dims(1, 2, 1024, 64, 64, 4, dtype="fp32")
    assert L.ssa_workspace_size(d32, L.SSA_OP_FULL_BWD) >= 3 * 2 * 1024 * 64 * 4


def _call(fn, dims, *args):
    return getattr(L.load(), fn)(ctypes.byref(dims) if dims is not None else None, *args)


BAD_DIMS = [
    (dict(B=0), L.SSA_ERR_INVALID_ARG),
    (dict(T=-64), L.SSA_ERR_INVALID_ARG),
    (dict(d=96), L.SSA_ERR_UNSUPPORTED),
    (dict(s=32), L.SSA_ERR_UNSUPPORTED),
    (dict(T=1000), L.SSA_ERR_UNSUPPORTED),      # T % s != 0
    (dict(k=0), L.SSA_ERR_INVALID_ARG),
    (dict(k=17), L.SSA_ERR_INVALID_ARG),        # k > nb
    (dict(dtype=7), L.SSA_ERR_INVALID_ARG),
    (dict(scale=0.0), L.SSA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), L.SSA_ERR_INVALID_ARG),
    (dict(T=64 * 300, k=257), L.SSA_ERR_UNSUPPORTED),                # slot index above the entry encoding
    (dict(B=1, H=512, T=131072, s=128, k=32), L.SSA_ERR_UNSUPPORTED),  # list positions beyond int32
    (dict(H=1, T=64 * 21000, k=256), L.SSA_ERR_UNSUPPORTED),         # index-fill staging beyond shared memory
]


BAD_DIMS += [
    (dict(H=6, Hkv=4), L.SSA_ERR_INVALID_ARG),                       # H not a multiple of Hkv
    (dict(H=6, Hkv=-1), L.SSA_ERR_INVALID_ARG),
    (dict(H=3, Hkv=1), L.SSA_ERR_UNSUPPORTED),                       # group of 3 does not divide a 128-row tile
]


@pytest.mark.parametrize("over,code", BAD_DIMS)
def test_dims_validation(lib, over, code):
    base = dict(B=1, H=2, T=1024, d=128, s=64, k=4, dtype=0, scale=0.088, Hkv=0)
    base.update(over)
    d = L.Dims(base["B"], base["H"], base["T"], base["d"], base["s"], base["k"], base["dtype"], base["scale"],
               base["Hkv"])
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    st = _call("ssa_sparse_attn_fwd", d, p, p, p, p, None, p, p, p, p, 1 << 40, None)
    assert st == code
    assert _call("ssa_sparse_index", d, p, p, 1 << 40, None) == code


def test_null_pointers_and_workspace(lib):
    d = L.make_dims(1, 2, 1024, 128, 64, 4)
    p = ctypes.c_void_p(16)
    assert _call("ssa_block_pool", None, p, p, None) == L.SSA_ERR_INVALID_ARG
    assert _call("ssa_block_pool", d, None, p, None) == L.SSA_ERR_INVALID_ARG
    assert _call("ssa_block_select", d, p, p, None, 1, None) == L.SSA_ERR_INVALID_ARG
    assert _call("ssa_block_select", d, p, p, p, 0, None) == L.SSA_ERR_UNSUPPORTED
    assert _call("ssa_block_select", d, p, p, p, 3, None) == L.SSA_ERR_UNSUPPORTED
    big = L.make_dims(1, 1, 2048 * 64, 128, 64, 4)     # nb = 2048 > 1024
    assert _call("ssa_block_select", big, p, p, p, 1, None) == L.SSA_ERR_UNSUPPORTED
    # short / missing / misaligned workspace or index
    need = L.ssa_workspace_size(d, L.SSA_OP_SPARSE_FWD)
    assert _call("ssa_sparse_attn_fwd", d, p, p, p, p, None, p, None, p, None, need, None) == L.SSA_ERR_WORKSPACE
    assert _call("ssa_sparse_attn_fwd", d, p, p, p, p, None, p, None, p, p, need - 1, None) == L.SSA_ERR_WORKSPACE
    assert _call("ssa_sparse_attn_fwd", d, p, p, p, p, None, p, None, p, ctypes.c_void_p(24), need,
                 None) == L.SSA_ERR_WORKSPACE
    assert _call("ssa_sparse_attn_fwd", d, p, p, p, p, ctypes.c_void_p(24), p, None, p, p, need,
                 None) == L.SSA_ERR_WORKSPACE
    need_i = L.ssa_workspace_size(d, L.SSA_OP_SPARSE_INDEX)
    assert _call("ssa_sparse_index", d, p, p, need_i - 1, None) == L.SSA_ERR_WORKSPACE
    assert _call("ssa_sparse_index", d, None, p, need_i, None) == L.SSA_ERR_INVALID_ARG
    need_s = L.ssa_workspace_size(d, L.SSA_OP_SPARSE_BWD)
    assert _call("ssa_sparse_attn_bwd", d, p, p, p, p, None, p, p, p, None, p, p, p, 0, p, need_s - 16,
                 None) == L.SSA_ERR_WORKSPACE
    need_b = L.ssa_workspace_size(d, L.SSA_OP_FULL_BWD)
    assert _call("ssa_full_attn_bwd", d, p, p, p, p, None, p, p, p, p, p, 0, p, need_b - 16,
                 None) == L.SSA_ERR_WORKSPACE
    assert _call("ssa_align_loss_fwd", d, p, p, 0, ctypes.c_float(0.0), ctypes.c_float(1), ctypes.c_float(1), p, p,
                 1 << 20, None) == L.SSA_ERR_INVALID_ARG
    assert _call("ssa_align_loss_fwd", d, p, p, 2, ctypes.c_float(1.0), ctypes.c_float(1), ctypes.c_float(1), p, p,
                 1 << 20, None) == L.SSA_ERR_INVALID_ARG          # unknown kind
    assert _call("ssa_align_loss_bwd", d, p, p, 0, ctypes.c_float(1.0), ctypes.c_float(1), ctypes.c_float(1), None,
                 p, p, 0, None) == L.SSA_ERR_INVALID_ARG
    assert _call("ssa_dropped_mass", d, p, None, p, None) == L.SSA_ERR_INVALID_ARG
    # the decode bulk-copies cache blocks: a cache base off a 16-byte boundary is refused
    odd = ctypes.c_void_p(24)
    assert _call("ssa_sparse_decode", d, p, p, odd, p, p, p, p, p, p, 1 << 40, None) == L.SSA_ERR_INVALID_ARG
    assert _call("ssa_sparse_decode", d, p, p, p, odd, p, p, p, p, p, 1 << 40, None) == L.SSA_ERR_INVALID_ARG


def test_binding_raises_on_error(lib):
    d = L.make_dims(1, 2, 1024, 128, 64, 4)
    with pytest.raises(L.SSAError) as e:
        L.ssa_block_pool(d, None, None, stream=0)
    assert e.value.status == L.SSA_ERR_INVALID_ARG


def test_build_flags_target_sm100a():
    flags = B.nvcc_flags()
    assert "arch=compute_100a,code=sm_100a" in flags and "-lineinfo" in flags


def test_product_does_not_import_oracle():
    pkg = os.path.join(ROOT, "block_top_sparse_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt and "ssa_oracle" not in txt, f


def test_decode_argument_validation(lib):
    """ssa_sparse_decode refuses what its kernels do not cover before enqueueing anything."""
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    big = 1 << 40

    def call(d, cache_len=p, q=p, kc=p, vc=p, kbar=p, idx=p, o=p, lse=p, ws=p, ws_bytes=big):
        return _call("ssa_sparse_decode", d, cache_len, q, kc, vc, kbar, idx, o, lse, ws, ws_bytes, None)

    ok = L.make_dims(2, 8, 4096, 128, 128, 4, Hkv=2)
    assert call(L.make_dims(2, 8, 4096, 64, 64, 4)) == L.SSA_ERR_UNSUPPORTED                  # d = 64
    assert call(L.make_dims(2, 8, 4096, 128, 128, 4, dtype="fp32")) == L.SSA_ERR_UNSUPPORTED   # fp32 caches
    assert call(L.make_dims(1, 32, 4096, 128, 128, 4, Hkv=1)) == L.SSA_ERR_UNSUPPORTED         # group of 32
    assert call(L.make_dims(1, 2, 128 * 1025, 128, 128, 4)) == L.SSA_ERR_UNSUPPORTED           # 1025 blocks
    for name in ("cache_len", "q", "kc", "vc", "kbar", "idx", "o", "lse"):
        assert call(ok, **{name: None}) == L.SSA_ERR_INVALID_ARG, name
    assert call(ok, q=ctypes.c_void_p(24)) == L.SSA_ERR_INVALID_ARG                            # q off 16 B
    need = L.ssa_workspace_size(ok, L.SSA_OP_DECODE)
    assert call(ok, ws_bytes=need - 1) == L.SSA_ERR_WORKSPACE
    assert call(ok, ws=None, ws_bytes=need) == L.SSA_ERR_WORKSPACE


def test_rope_argument_validation(lib):
    """ssa_rope refuses a bad base, factor, head count or start position before enqueueing anything."""
    p = ctypes.c_void_p(16)
    d = L.make_dims(1, 4, 1024, 128, 128, 1)
    f = ctypes.c_float

    def call(X=p, heads=4, pos0=0, base=10000.0, factor=1.0, dims=d):
        return _call("ssa_rope", dims, X, heads, pos0, f(base), f(factor), 0, None)

    for over in (dict(X=None), dict(heads=0), dict(pos0=-1), dict(base=1.0), dict(base=float("nan")),
                 dict(base=float("inf")), dict(factor=0.0), dict(factor=-4.0), dict(factor=float("inf"))):
        assert call(**over) == L.SSA_ERR_INVALID_ARG, over
    # B * heads * T rows beyond int32
    assert call(dims=L.make_dims(1, 1, 1 << 22, 128, 128, 1), heads=1024) == L.SSA_ERR_UNSUPPORTED

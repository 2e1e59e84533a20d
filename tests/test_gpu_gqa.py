"""Grouped-query attention (Hkv key/value heads shared by H / Hkv query heads each)
on the GPU against the fp64 oracle: pooling per key head, the shared per-group
selection (ranked by the sum of the group's scores), both attention streams
forward and backward (dK, dV summed over the group; exact gradients), and one
whole step in the benchmark's gradient mode.  Group sizes 2, 4 and 8 on the
tensor-core path and 2 on the CUDA-core fp32 path, with ragged T and -1 padded
selections."""
import numpy as np
import pytest

import oracle as ora
from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import inputs, ops

from .helpers import check_close, check_gpu_selection, to_device, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# (name, workload, overrides, Hkv, k)
CASES = [
    ("g2_train_ragged", "train", dict(B=1, H=4, T=704), 2, 4),
    ("g4_long_sink", "long", dict(H=8, T=1536), 2, 5),
    ("g8_prefill_planted", "prefill", dict(H=8, T=2048), 1, 16),
    ("g2_tiny_fp32", "tiny", dict(H=4, T=512), 2, 4),
]


@pytest.fixture(scope="module", autouse=True)
def _build():
    from block_top_sparse_b200 import build
    build.build()
    ora.build()


def _setup(wlname, over, Hkv, k):
    g = inputs.group_kv(inputs.generate(inputs.WORKLOADS[wlname], with_dO=True, **over), Hkv)
    w = g["wl"]
    BH, BHk = w.B * w.H, w.B * Hkv
    f = {key: inputs.to_float64(g[key], w.dtype).reshape((BHk if key in ("K", "V") else BH), w.T, w.d)
         for key in ("Q", "K", "V", "dO")}
    dims = L.make_dims(w.B, w.H, w.T, w.d, w.s, k, dtype=w.dtype, Hkv=Hkv)
    dev = {key: to_device(g[key], w.dtype) for key in ("Q", "K", "V", "dO")}
    return w, dims, f, dev


@pytest.mark.parametrize("name,wlname,over,Hkv,k", CASES, ids=[c[0] for c in CASES])
def test_gqa_pool_select(name, wlname, over, Hkv, k):
    w, dims, f, dev = _setup(wlname, over, Hkv, k)
    Kbar = ops.block_pool(dims, dev["K"])
    Kbar_ref = ora.block_pool(f["K"], w.s)
    np.testing.assert_allclose(to_np(Kbar).reshape(Kbar_ref.shape), Kbar_ref, rtol=2e-6, atol=1e-7)
    idx = ops.block_select(dims, dev["Q"], Kbar)
    torch.cuda.synchronize()
    check_gpu_selection(ora, "gqa." + name, idx.cpu().numpy().reshape(w.B * Hkv, w.T, k), f["Q"], Kbar_ref, w.s, k)
    assert L.ssa_get_device_error() == L.SSA_OK


@pytest.mark.parametrize("stream", ["full", "sparse"])
@pytest.mark.parametrize("name,wlname,over,Hkv,k", CASES, ids=[c[0] for c in CASES])
def test_gqa_attention(name, wlname, over, Hkv, k, stream):
    w, dims, f, dev = _setup(wlname, over, Hkv, k)
    bf16 = w.dtype == "bf16"
    BH, BHk = w.B * w.H, w.B * Hkv
    idx_ref = None
    idx_dev = index = None
    if stream == "sparse":
        idx_ref, _, _ = ora.block_select(f["Q"], ora.block_pool(f["K"], w.s), w.s, k)
        idx_dev = torch.from_numpy(idx_ref.reshape(w.B, Hkv, w.T, k)).cuda()
        index = ops.sparse_index(dims, idx_dev)
    O, lse, O_lo = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"], idx_dev, index=index)
    O_ref, lse_ref = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, dims.scale, idx_ref)
    tag = "gqa.%s.%s" % (name, stream)
    check_close(tag + ".O", to_np(O).reshape(BH, w.T, w.d), O_ref, bf16)
    np.testing.assert_allclose(to_np(lse).reshape(BH, w.T), lse_ref, rtol=0, atol=2e-3)
    gref = ora.attn_bwd(f["Q"], f["K"], f["V"], f["dO"], w.s, dims.scale, idx_ref)
    dQ, dK, dV = ops.attn_bwd(dims, dev["Q"], dev["K"], dev["V"], O, lse, dev["dO"], idx_dev, O_lo=O_lo, index=index)
    assert tuple(dK.shape) == (w.B, Hkv, w.T, w.d) and tuple(dV.shape) == (w.B, Hkv, w.T, w.d)
    check_close(tag + ".dQ", to_np(dQ).reshape(BH, w.T, w.d), gref[0], bf16)
    check_close(tag + ".dK", to_np(dK).reshape(BHk, w.T, w.d), gref[1], bf16)
    check_close(tag + ".dV", to_np(dV).reshape(BHk, w.T, w.d), gref[2], bf16)
    assert L.ssa_get_device_error() == L.SSA_OK


@pytest.mark.parametrize("main", ["full", "sparse"])
def test_gqa_step(main):
    """The whole step (both streams, alignment, fp32 gradients of both streams summed) with Hkv = 2, G = 4."""
    w, dims, f, dev = _setup("long", dict(H=8, T=1024), 2, 4)
    BH, BHk = w.B * w.H, w.B * 2
    step = ops.SSAStep(dims, main=main, grad_fp32=True)
    step.forward(dev["Q"], dev["K"], dev["V"])
    step.main_grad_buffer().copy_(dev["dO"])
    step.backward(dev["Q"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    Kbar = ora.block_pool(f["K"], w.s)
    sel = step.idx.cpu().numpy().reshape(BHk, w.T, 4)
    check_gpu_selection(ora, "gqa.step." + main, sel, f["Q"], Kbar, w.s, 4)
    Of_ref, _ = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, dims.scale)
    Os_ref, _ = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, dims.scale, sel)
    check_close("gqa.step.Of", to_np(step.Of).reshape(BH, w.T, w.d), Of_ref, True)
    check_close("gqa.step.Os", to_np(step.Os).reshape(BH, w.T, w.d), Os_ref, True)
    gf, gs = ora.align_bwd(Of_ref, Os_ref)
    dOf = f["dO"] + gf if main == "full" else gf
    dOs = f["dO"] + gs if main == "sparse" else gs
    a = ora.attn_bwd(f["Q"], f["K"], f["V"], dOf, w.s, dims.scale)
    b = ora.attn_bwd(f["Q"], f["K"], f["V"], dOs, w.s, dims.scale, sel)
    for nm, g, ra, rb, nh in zip(("dQ", "dK", "dV"), (step.dQ, step.dK, step.dV), a, b, (BH, BHk, BHk)):
        check_close("gqa.step.%s.%s" % (main, nm), to_np(g).reshape(nh, w.T, w.d), ra + rb, False)
    assert L.ssa_get_device_error() == L.SSA_OK

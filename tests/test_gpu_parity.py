"""GPU parity: every step of the path through the C ABI against the fp64 oracle,
on seeded inputs at sizes the oracle finishes in seconds that still span several
tiles and a ragged tail (T not a multiple of the 128-row tile, lists whose
length is not a multiple of 128, -1 padded selections, k = 1 and k = nb, a single
block, many short heads)."""
import numpy as np
import pytest

import oracle as ora
from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import inputs, ops

from .helpers import bf16_half_ulp, check_close, selection_report, to_device, to_np, workload_arrays

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# (name, workload, overrides, k)
CASES = [
    ("tiny_fp32_d64", "tiny", dict(), 4),
    ("train_ragged_s64", "train", dict(B=1, H=2, T=704), 4),
    ("train_s64_k8", "train", dict(B=2, H=1, T=1024), 8),
    ("long_s128_sink", "long", dict(H=2, T=1536), 5),
    ("prefill_planted", "prefill", dict(H=2, T=2048), 16),
    ("k_equals_nb", "train", dict(B=1, H=1, T=512), 8),
    ("k_one", "long", dict(H=1, T=1024), 1),
    ("single_block", "long", dict(H=1, T=128), 1),  # nb = 1: every query attends its own block only
    ("many_heads_short", "long", dict(B=2, H=8, T=384), 3),
]


def _setup(wlname, over, k):
    wl = inputs.WORKLOADS[wlname]
    f, g, w = workload_arrays(wl, with_dO=True, **over)
    dims = L.make_dims(w.B, w.H, w.T, w.d, w.s, k, dtype=w.dtype)
    dev = {key: to_device(g[key], w.dtype) for key in ("Q", "K", "V", "dO")}
    return w, dims, f, dev


@pytest.fixture(scope="module", autouse=True)
def _build():
    from block_top_sparse_b200 import build
    build.build()
    ora.build()


@pytest.mark.parametrize("name,wlname,over,k", CASES, ids=[c[0] for c in CASES])
def test_pool_select(name, wlname, over, k):
    w, dims, f, dev = _setup(wlname, over, k)
    Kbar = ops.block_pool(dims, dev["K"])
    Kbar_ref = ora.block_pool(f["K"], w.s)
    got = to_np(Kbar).reshape(Kbar_ref.shape)
    np.testing.assert_allclose(got, Kbar_ref, rtol=2e-6, atol=1e-7)
    idx = ops.block_select(dims, dev["Q"], Kbar)
    torch.cuda.synchronize()
    idx_ref, r1, r2 = ora.block_select(f["Q"], Kbar_ref, w.s, k)
    got_idx = idx.cpu().numpy().reshape(idx_ref.shape)
    assert ora.check_selection(got_idx, w.s)
    rep = selection_report(got_idx, idx_ref, r1, r2)
    assert rep["mismatch"] == 0, rep
    assert L.ssa_get_device_error() == L.SSA_OK


def _attn_check(w, dims, f, dev, idx_ref, tag):
    bf16 = w.dtype == "bf16"
    BH = w.B * w.H
    scale = dims.scale
    idx_dev = None if idx_ref is None else torch.from_numpy(idx_ref.reshape(w.B, w.H, w.T, -1)).cuda()
    O, lse = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"], idx_dev)
    O_ref, lse_ref = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, scale, idx_ref)
    check_close(tag + ".O", to_np(O).reshape(BH, w.T, w.d), O_ref, bf16)
    np.testing.assert_allclose(to_np(lse).reshape(BH, w.T), lse_ref, rtol=0, atol=2e-3)
    dQ, dK, dV = ops.attn_bwd(dims, dev["Q"], dev["K"], dev["V"], O, lse, dev["dO"], idx_dev)
    # the backward is given the forward's output as stored: D = dO . o with o in the output dtype
    gref = ora.attn_bwd(f["Q"], f["K"], f["V"], f["dO"], w.s, scale, idx_ref, stored_o="bf16" if bf16 else "exact")
    for nm, g, r in zip(("dQ", "dK", "dV"), (dQ, dK, dV), gref):
        check_close(tag + "." + nm, to_np(g).reshape(BH, w.T, w.d), r, bf16)
    assert L.ssa_get_device_error() == L.SSA_OK


@pytest.mark.parametrize("name,wlname,over,k", CASES, ids=[c[0] for c in CASES])
def test_full_attention(name, wlname, over, k):
    w, dims, f, dev = _setup(wlname, over, k)
    _attn_check(w, dims, f, dev, None, name + ".full")


@pytest.mark.parametrize("name,wlname,over,k", CASES, ids=[c[0] for c in CASES])
def test_sparse_attention(name, wlname, over, k):
    # Both sides attend over the oracle's selection, so the attention kernels are
    # compared on identical inputs (selection parity is tested separately).
    w, dims, f, dev = _setup(wlname, over, k)
    idx_ref, _, _ = ora.block_select(f["Q"], ora.block_pool(f["K"], w.s), w.s, k)
    _attn_check(w, dims, f, dev, idx_ref, name + ".sparse")


def test_sparse_equals_full_when_k_covers_all_blocks():
    w, dims, f, dev = _setup("train", dict(B=1, H=2, T=768), 12)
    idx = ops.block_select(dims, dev["Q"], ops.block_pool(dims, dev["K"]))
    Os, ls = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"], idx)
    Of, lf = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"])
    # same attended set; the two kernels sum in different orders
    np.testing.assert_allclose(to_np(Os), to_np(Of), rtol=0, atol=2 ** -7)
    np.testing.assert_allclose(to_np(ls), to_np(lf), rtol=0, atol=1e-4)
    delta = ops.dropped_mass(dims, ls, lf)
    assert float(delta.abs().max()) < 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_align_loss(dtype):
    rng = np.random.default_rng(7)
    shape = (2, 3, 256, 128)
    of = rng.standard_normal(shape).astype(np.float32) * 0.8
    os_ = of + rng.standard_normal(shape).astype(np.float32) * 0.9
    raw_f = inputs.f32_to_bf16_bits(of) if dtype == "bf16" else of
    raw_s = inputs.f32_to_bf16_bits(os_) if dtype == "bf16" else os_
    Of, Os = to_device(raw_f, dtype), to_device(raw_s, dtype)
    dims = L.make_dims(2, 3, 256, 128, 64, 1, dtype=dtype)
    f64 = lambda a: inputs.to_float64(a, dtype)  # noqa: E731
    for beta, ws, wc in ((1.0, 1.0, 1.0), (0.5, 0.25, 2.0)):
        loss = ops.align_fwd(dims, Of, Os, beta, ws, wc)
        ref = ora.align_fwd(f64(raw_f), f64(raw_s), beta, ws, wc)
        assert float(loss) == pytest.approx(ref, rel=1e-5)
        g = torch.full((), 1.5, dtype=torch.float32, device="cuda")
        dOf, dOs = ops.align_bwd(dims, Of, Os, g, beta, ws, wc)
        rf, rs = ora.align_bwd(f64(raw_f), f64(raw_s), beta, ws, wc, 1.5)
        for got, ref in ((dOf, rf), (dOs, rs)):
            # elementwise result: fp32 arithmetic, then one rounding to the output type
            allow = bf16_half_ulp(ref) if dtype == "bf16" else 0.0
            assert np.all(np.abs(to_np(got) - ref) <= allow + 1e-5 * np.abs(ref) + 1e-12)
        # accumulate bits: only dOf receives the add
        base = torch.ones_like(Of)
        dOs2 = torch.zeros_like(Os)
        ops.align_bwd(dims, Of, Os, g, beta, ws, wc, dOf=base, dOs=dOs2, accumulate=L.SSA_ACC_OF)
        np.testing.assert_allclose(to_np(base) - 1.0, to_np(dOf), rtol=0, atol=2e-2 * np.abs(rf).max() + 1e-2)
        np.testing.assert_allclose(to_np(dOs2), to_np(dOs), rtol=0, atol=0)


def test_dropped_mass_matches_oracle_and_bound():
    w, dims, f, dev = _setup("prefill", dict(H=2, T=2048), 4)
    idx_np, _, _ = ora.block_select(f["Q"], ora.block_pool(f["K"], w.s), w.s, 4)
    idx = torch.from_numpy(idx_np.reshape(w.B, w.H, w.T, 4)).cuda()
    Os, ls = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"], idx)
    Of, lf = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"])
    delta = to_np(ops.dropped_mass(dims, ls, lf)).reshape(-1, w.T)
    _, ls_ref = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, dims.scale, idx_np)
    _, lf_ref = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, dims.scale)
    np.testing.assert_allclose(delta, ora.dropped_mass(ls_ref, lf_ref), rtol=0, atol=5e-3)
    # Appendix B bound on the GPU outputs: |o_f - o_s| <= 2 delta max|v| (+ bf16 rounding of both outputs)
    vmax = np.linalg.norm(f["V"], axis=-1).max()
    gap = np.linalg.norm(to_np(Of) - to_np(Os), axis=-1).reshape(-1, w.T)
    assert np.all(gap <= 2 * np.maximum(delta, 0) * vmax + 2e-2)


def test_step_both_streams_matches_oracle():
    """One training step (pool, select, both attentions, alignment, all grads) vs the oracle chain."""
    w, dims, f, dev = _setup("train", dict(B=1, H=2, T=1024), 8)
    for main in ("full", "sparse"):
        step = ops.SSAStep(dims, main=main)
        step.forward(dev["Q"], dev["K"], dev["V"])
        step.main_grad_buffer().copy_(dev["dO"])
        step.backward(dev["Q"], dev["K"], dev["V"])
        torch.cuda.synchronize()
        s, scale = w.s, dims.scale
        Kbar = ora.block_pool(f["K"], s)
        idx_ref, r1, r2 = ora.block_select(f["Q"], Kbar, s, 8)
        got_idx = step.idx.cpu().numpy().reshape(idx_ref.shape)
        rep = selection_report(got_idx, idx_ref, r1, r2)
        assert rep["mismatch"] == 0, rep
        same = ~np.any(got_idx != idx_ref, axis=-1)
        Of_ref, _ = ora.attn_fwd(f["Q"], f["K"], f["V"], s, scale)
        Os_ref, _ = ora.attn_fwd(f["Q"], f["K"], f["V"], s, scale, idx_ref)
        check_close("step.Of", to_np(step.Of).reshape(Of_ref.shape), Of_ref, True)
        check_close("step.Os", to_np(step.Os).reshape(Os_ref.shape)[same], Os_ref[same], True)
        loss_ref = ora.align_fwd(Of_ref, Os_ref)
        assert float(step.loss) == pytest.approx(loss_ref, rel=2e-2, abs=1e-5)
        gf, gs = ora.align_bwd(Of_ref, Os_ref)
        dOf = f["dO"] + gf if main == "full" else gf
        dOs = f["dO"] + gs if main == "sparse" else gs
        g_full = ora.attn_bwd(f["Q"], f["K"], f["V"], dOf, s, scale, stored_o="bf16")
        g_sparse = ora.attn_bwd(f["Q"], f["K"], f["V"], dOs, s, scale, idx_ref, stored_o="bf16")
        if rep["differ"] == 0:
            for nm, g, a, b in zip(("dQ", "dK", "dV"), (step.dQ, step.dK, step.dV), g_full, g_sparse):
                check_close("step.%s.%s" % (main, nm), to_np(g).reshape(a.shape), a + b, True)
    assert L.ssa_get_device_error() == L.SSA_OK


@pytest.mark.parametrize("name,wlname,over,k", [CASES[1], CASES[3]], ids=[CASES[1][0], CASES[3][0]])
def test_attention_at_unit_scale(name, wlname, over, k):
    # The other reading of the softmax scale: the inputs' d^-1/4 already folds it in (unit-variance logits).
    w, _, f, dev = _setup(wlname, over, k)
    dims = L.make_dims(w.B, w.H, w.T, w.d, w.s, k, dtype=w.dtype, scale=1.0)
    Kbar = ora.block_pool(f["K"], w.s)
    idx_ref, _, _ = ora.block_select(f["Q"], Kbar, w.s, k)
    _attn_check(w, dims, f, dev, None, name + ".unit_scale.full")
    _attn_check(w, dims, f, dev, idx_ref, name + ".unit_scale.sparse")

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

from .helpers import (bf16_half_ulp, check_close, check_gpu_selection, log_result, rel_l2, to_device, to_np,
                      workload_arrays)

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
    check_gpu_selection(ora, name, idx.cpu().numpy().reshape(w.B * w.H, w.T, k), f["Q"], Kbar_ref, w.s, k)
    assert L.ssa_get_device_error() == L.SSA_OK


def _attn_check(w, dims, f, dev, idx_ref, tag):
    """Forward and backward of one stream against the fp64 oracle on the same inputs (and selection).

    Gradients are compared with the exact gradient of the pages' definition (D_t = dO_t . o_t with the
    exact o_t).  The backward is given the forward's bf16 output together with its rounding residual
    O_lo; the errors of the form that uses the bf16 output alone are logged for the record."""
    bf16 = w.dtype == "bf16"
    BH = w.B * w.H
    scale = dims.scale
    idx_dev = None if idx_ref is None else torch.from_numpy(idx_ref.reshape(w.B, w.H, w.T, -1)).cuda()
    index = None if idx_dev is None else ops.sparse_index(dims, idx_dev)
    O, lse, O_lo = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"], idx_dev, index=index)
    O_ref, lse_ref = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, scale, idx_ref)
    got_O = to_np(O).reshape(BH, w.T, w.d)
    check_close(tag + ".O", got_O, O_ref, bf16)
    np.testing.assert_allclose(to_np(lse).reshape(BH, w.T), lse_ref, rtol=0, atol=2e-3)
    if O_lo is not None:
        lo = to_np(O_lo).reshape(BH, w.T, w.d)
        # a rounding residual: at most half a bf16 ulp of the stored output, and O + O_lo is closer
        assert np.all(np.abs(lo) <= bf16_half_ulp(got_O) + 1e-30)
        full_prec = got_O + lo
        check_close(tag + ".O+O_lo", full_prec, O_ref, False)
        assert rel_l2(full_prec, O_ref) <= rel_l2(got_O, O_ref) + 1e-6
    gref = ora.attn_bwd(f["Q"], f["K"], f["V"], f["dO"], w.s, scale, idx_ref)
    grads = ops.attn_bwd(dims, dev["Q"], dev["K"], dev["V"], O, lse, dev["dO"], idx_dev, O_lo=O_lo, index=index)
    for nm, g, r in zip(("dQ", "dK", "dV"), grads, gref):
        check_close(tag + "." + nm, to_np(g).reshape(BH, w.T, w.d), r, bf16)
    if bf16:
        # diagnostic only: the same backward given the bf16 output alone
        g2 = ops.attn_bwd(dims, dev["Q"], dev["K"], dev["V"], O, lse, dev["dO"], idx_dev, index=index)
        for nm, g, r in zip(("dQ", "dK", "dV"), g2, gref):
            log_result(tag + "." + nm + ".without_O_lo", {"rel_l2": rel_l2(to_np(g).reshape(BH, w.T, w.d), r)})
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
    Os, ls, _ = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"], idx)
    Of, lf, _ = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"])
    # same attended set; the two kernels sum in different orders
    np.testing.assert_allclose(to_np(Os), to_np(Of), rtol=0, atol=2 ** -7)
    np.testing.assert_allclose(to_np(ls), to_np(lf), rtol=0, atol=1e-4)
    delta = ops.dropped_mass(dims, ls, lf)
    assert float(delta.abs().max()) < 1e-4


@pytest.mark.parametrize("kind", ["smooth_l1", "l2"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_align_loss(dtype, kind):
    rng = np.random.default_rng(7)
    shape = (2, 3, 256, 128)
    of = rng.standard_normal(shape).astype(np.float32) * 0.8
    os_ = of + rng.standard_normal(shape).astype(np.float32) * 0.9
    raw_f = inputs.f32_to_bf16_bits(of) if dtype == "bf16" else of
    raw_s = inputs.f32_to_bf16_bits(os_) if dtype == "bf16" else os_
    Of, Os = to_device(raw_f, dtype), to_device(raw_s, dtype)
    dims = L.make_dims(2, 3, 256, 128, 64, 1, dtype=dtype)
    f64 = lambda a: inputs.to_float64(a, dtype)  # noqa: E731
    kc = {"smooth_l1": L.SSA_ALIGN_SMOOTH_L1, "l2": L.SSA_ALIGN_L2}[kind]
    for beta, ws, wc in ((1.0, 1.0, 1.0), (0.5, 0.25, 2.0)):
        loss = ops.align_fwd(dims, Of, Os, beta, ws, wc, kind=kc)
        ref = ora.align_fwd(f64(raw_f), f64(raw_s), beta, ws, wc, kind=kind)
        assert float(loss) == pytest.approx(ref, rel=1e-5)
        g = torch.full((), 1.5, dtype=torch.float32, device="cuda")
        dOf, dOs = ops.align_bwd(dims, Of, Os, g, beta, ws, wc, kind=kc)
        rf, rs = ora.align_bwd(f64(raw_f), f64(raw_s), beta, ws, wc, 1.5, kind=kind)
        for got, ref in ((dOf, rf), (dOs, rs)):
            # elementwise result: fp32 arithmetic, then one rounding to the output type
            allow = bf16_half_ulp(ref) if dtype == "bf16" else 0.0
            assert np.all(np.abs(to_np(got) - ref) <= allow + 1e-5 * np.abs(ref) + 1e-12)
        # accumulate bits: only dOf receives the add
        base = torch.ones_like(Of)
        dOs2 = torch.zeros_like(Os)
        ops.align_bwd(dims, Of, Os, g, beta, ws, wc, dOf=base, dOs=dOs2, accumulate=L.SSA_ACC_OF, kind=kc)
        np.testing.assert_allclose(to_np(base) - 1.0, to_np(dOf), rtol=0, atol=2e-2 * np.abs(rf).max() + 1e-2)
        np.testing.assert_allclose(to_np(dOs2), to_np(dOs), rtol=0, atol=0)


def test_dropped_mass_matches_oracle_and_bound():
    w, dims, f, dev = _setup("prefill", dict(H=2, T=2048), 4)
    idx_np, _, _ = ora.block_select(f["Q"], ora.block_pool(f["K"], w.s), w.s, 4)
    idx = torch.from_numpy(idx_np.reshape(w.B, w.H, w.T, 4)).cuda()
    Os, ls, _ = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"], idx)
    Of, lf, _ = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"])
    delta = to_np(ops.dropped_mass(dims, ls, lf)).reshape(-1, w.T)
    _, ls_ref = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, dims.scale, idx_np)
    _, lf_ref = ora.attn_fwd(f["Q"], f["K"], f["V"], w.s, dims.scale)
    np.testing.assert_allclose(delta, ora.dropped_mass(ls_ref, lf_ref), rtol=0, atol=5e-3)
    # Appendix B bound on the GPU outputs: |o_f - o_s| <= 2 delta max|v| (+ bf16 rounding of both outputs)
    vmax = np.linalg.norm(f["V"], axis=-1).max()
    gap = np.linalg.norm(to_np(Of) - to_np(Os), axis=-1).reshape(-1, w.T)
    assert np.all(gap <= 2 * np.maximum(delta, 0) * vmax + 2e-2)


def test_step_both_streams_matches_oracle():
    """One training step (pool, select, both attentions, alignment, all grads) vs the oracle chain.

    The selection is checked first (bit-exact apart from near-tie rows, which must still be valid top
    sets); the oracle then runs the sparse stream on the selection the GPU made, so every row of every
    output and gradient is compared whatever the near-tie rows chose."""
    w, dims, f, dev = _setup("train", dict(B=1, H=2, T=1024), 8)
    for main in ("full", "sparse"):
        step = ops.SSAStep(dims, main=main)
        step.forward(dev["Q"], dev["K"], dev["V"])
        step.main_grad_buffer().copy_(dev["dO"])
        step.backward(dev["Q"], dev["K"], dev["V"])
        torch.cuda.synchronize()
        s, scale = w.s, dims.scale
        Kbar = ora.block_pool(f["K"], s)
        got_idx = step.idx.cpu().numpy().reshape(w.B * w.H, w.T, 8)
        check_gpu_selection(ora, "step." + main, got_idx, f["Q"], Kbar, s, 8)
        Of_ref, _ = ora.attn_fwd(f["Q"], f["K"], f["V"], s, scale)
        Os_ref, _ = ora.attn_fwd(f["Q"], f["K"], f["V"], s, scale, got_idx)
        check_close("step.Of", to_np(step.Of).reshape(Of_ref.shape), Of_ref, True)
        check_close("step.Os", to_np(step.Os).reshape(Os_ref.shape), Os_ref, True)
        loss_ref = ora.align_fwd(Of_ref, Os_ref)
        assert float(step.loss) == pytest.approx(loss_ref, rel=2e-2, abs=1e-5)
        gf, gs = ora.align_bwd(Of_ref, Os_ref)
        dOf = f["dO"] + gf if main == "full" else gf
        dOs = f["dO"] + gs if main == "sparse" else gs
        g_full = ora.attn_bwd(f["Q"], f["K"], f["V"], dOf, s, scale)
        g_sparse = ora.attn_bwd(f["Q"], f["K"], f["V"], dOs, s, scale, got_idx)
        for nm, g, a, b in zip(("dQ", "dK", "dV"), (step.dQ, step.dK, step.dV), g_full, g_sparse):
            check_close("step.%s.%s" % (main, nm), to_np(g).reshape(a.shape), a + b, True)
    assert L.ssa_get_device_error() == L.SSA_OK


@pytest.mark.parametrize("name,wlname,over,k", [CASES[0], CASES[1], CASES[3]], ids=[CASES[0][0], CASES[1][0], CASES[3][0]])
def test_fp32_gradients(name, wlname, over, k):
    """SSA_BWD_GRAD_FP32: dQ, dK, dV written (and accumulated) in fp32; both streams against the oracle, then
    the sparse stream added onto the full stream's fp32 gradients (the step's order) against their sum.

    The gradients are products of bf16 tensor-core operands (P, dS, Q, K, V, dO), so they are held to the bar
    of the bf16-stored result (max-abs 1e-2 beyond half a bf16 ulp of the value, rel-L2 5e-3): the fp32
    storage removes the final rounding, not the operands' precision."""
    w, dims, f, dev = _setup(wlname, over, k)
    BH = w.B * w.H
    idx_ref, _, _ = ora.block_select(f["Q"], ora.block_pool(f["K"], w.s), w.s, k)
    idx_dev = torch.from_numpy(idx_ref.reshape(w.B, w.H, w.T, -1)).cuda()
    Of, lf, Of_lo = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"])
    Os, ls, Os_lo = ops.attn_fwd(dims, dev["Q"], dev["K"], dev["V"], idx_dev)
    g_full = ora.attn_bwd(f["Q"], f["K"], f["V"], f["dO"], w.s, dims.scale)
    g_sp = ora.attn_bwd(f["Q"], f["K"], f["V"], f["dO"], w.s, dims.scale, idx_ref)
    grads = ops.attn_bwd(dims, dev["Q"], dev["K"], dev["V"], Of, lf, dev["dO"], O_lo=Of_lo, grad_fp32=True)
    assert all(g.dtype == torch.float32 for g in grads)
    for nm, g, r in zip(("dQ", "dK", "dV"), grads, g_full):
        check_close(name + ".fp32grad.full." + nm, to_np(g).reshape(BH, w.T, w.d), r, w.dtype == "bf16")
    ops.attn_bwd(dims, dev["Q"], dev["K"], dev["V"], Os, ls, dev["dO"], idx_dev, grads=grads, O_lo=Os_lo,
                 grad_fp32=True)
    for nm, g, a, b in zip(("dQ", "dK", "dV"), grads, g_full, g_sp):
        check_close(name + ".fp32grad.sum." + nm, to_np(g).reshape(BH, w.T, w.d), a + b, w.dtype == "bf16")
    assert L.ssa_get_device_error() == L.SSA_OK


def test_sparse_forward_with_values_beyond_fp16_range():
    """Blocks whose |v| reaches 2^15 keep their partial outputs in range by a power-of-two exponent that the
    merge restores: values up to 2^20 attended alongside ordinary ones."""
    w, dims, f, dev = _setup("long", dict(H=2, T=1024), 4)
    raw = inputs.generate(inputs.WORKLOADS["long"], H=2, T=1024)["V"].copy()
    V = inputs.to_float64(raw, "bf16").reshape(2, 1024, 128)
    V[0, 128:256] *= 2.0 ** 20  # block 1 of head 0
    V[1, 640:768] *= 2.0 ** 16  # block 5 of head 1
    Vb = inputs.f32_to_bf16_bits(V.astype(np.float32))
    Vd = to_device(Vb, "bf16")
    Vf = inputs.to_float64(Vb, "bf16").reshape(2, 1024, 128)
    idx_ref, _, _ = ora.block_select(f["Q"], ora.block_pool(f["K"], w.s), w.s, 4)
    idx_dev = torch.from_numpy(idx_ref.reshape(1, 2, 1024, 4)).cuda()
    O, lse, O_lo = ops.attn_fwd(dims, dev["Q"], dev["K"], Vd, idx_dev)
    O_ref, lse_ref = ora.attn_fwd(f["Q"], f["K"], Vf, w.s, dims.scale, idx_ref)
    got = to_np(O).reshape(2, 1024, 128)
    assert np.all(np.isfinite(got))
    rel = np.linalg.norm(got - O_ref) / np.linalg.norm(O_ref)
    assert rel < 5e-3, rel
    np.testing.assert_allclose(to_np(lse).reshape(2, 1024), lse_ref, rtol=0, atol=2e-3)
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

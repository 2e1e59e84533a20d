"""Full-size parity: every workload at its real size, in the launch configuration
the benchmark times (SSAStep over the whole path, fp32 gradients), checked against the fp64
oracle on sampled outputs it can compute one by one:
  * selection: every row of every head bit-exact apart from near-tie rows, each
    of which must still be a valid top set (tests/helpers.check_gpu_selection);
  * forward outputs and lse of both streams on sampled query rows, the sparse
    stream on the selection the GPU made (checked above), so no row is skipped;
  * gradients (training workloads): dQ on sampled query rows, dK and dV on
    sampled key rows, of the sampled heads, with the seeded dO routed to the
    full stream (4K, 32K) or the sparse stream (32K), against the exact
    gradient (D_t = dO_t . o_t with the exact o_t);
  * the dropped mass on sampled rows, and the bound |o_f - o_s| <= 2 delta max|v|
    on every row of every head (a property that holds at any size).
"""
import numpy as np
import pytest

import oracle as ora
from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import inputs, ops

from .helpers import check_close, check_gpu_selection, to_device, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _rows(T, n, seed):
    rng = np.random.default_rng(seed)
    r = set(rng.choice(T, size=n, replace=False).tolist())
    r.update([0, 1, T // 2, T - 2, T - 1])
    return np.array(sorted(r), dtype=np.int64)


_CACHE = {}


def _inputs(wlname, backward):
    if wlname not in _CACHE:
        _CACHE.clear()
        _CACHE[wlname] = inputs.generate(inputs.WORKLOADS[wlname], with_dO=backward)
    return _CACHE[wlname]


def _pick(t, B, H, T, bh, rows=None):
    x = t.reshape(B * H, T, -1)[bh]
    if rows is not None:
        x = x[torch.from_numpy(rows).to(x.device)]
    return to_np(x)[None]


def _run(wlname, k, heads, n_rows, backward, main="full"):
    g = _inputs(wlname, backward)
    w = g["wl"]
    B, H, T, d, s = w.B, w.H, w.T, w.d, w.s
    dims = L.make_dims(B, H, T, d, s, k)
    dev = {key: to_device(g[key], "bf16") for key in ("Q", "K", "V") + (("dO",) if backward else ())}
    step = ops.SSAStep(dims, main=main, grad_fp32=True)  # the benchmark's gradient mode
    step.forward(dev["Q"], dev["K"], dev["V"])
    if backward:
        step.main_grad_buffer().copy_(dev["dO"])
        step.backward(dev["Q"], dev["K"], dev["V"])
    delta = ops.dropped_mass(dims, step.lse_s, step.lse_f)
    torch.cuda.synchronize()
    assert L.ssa_get_device_error() == L.SSA_OK

    idx_all = step.idx.cpu().numpy().reshape(B * H, T, k)
    # property at any size: |o_f - o_s| <= 2 delta max|v| (+ rounding of the two bf16 outputs)
    Of_all, Os_all = step.Of.float(), step.Os.float()
    gap = torch.linalg.vector_norm(Of_all - Os_all, dim=-1)
    vmax = torch.linalg.vector_norm(dev["V"].float(), dim=-1).amax(dim=-1, keepdim=True)
    slack = 2 * delta.clamp(min=0) * vmax + 2e-2
    assert bool((gap <= slack).all())

    # selection of every head against the oracle
    Qall = inputs.to_float64(g["Q"].reshape(B * H, T, d), "bf16")
    Kbar_all = ora.block_pool(inputs.to_float64(g["K"].reshape(B * H, T, d), "bf16"), s)
    np.testing.assert_allclose(step.Kbar.cpu().numpy().reshape(Kbar_all.shape), Kbar_all, rtol=2e-6, atol=1e-7)
    report = check_gpu_selection(ora, "%s.k%d" % (wlname, k), idx_all, Qall, Kbar_all, s, k)
    del Qall

    rows = _rows(T, n_rows, 11)
    for bh in heads:
        sl = slice(bh, bh + 1)
        f = {key: inputs.to_float64(g[key].reshape(B * H, T, d)[sl], "bf16") for key in ("Q", "K", "V", "dO")
             if key in dev}
        sel = idx_all[sl]  # the GPU's selection, checked above
        Of, lf = ora.attn_fwd(f["Q"], f["K"], f["V"], s, dims.scale, rows=rows)
        Os, ls = ora.attn_fwd(f["Q"], f["K"], f["V"], s, dims.scale, sel, rows=rows)
        check_close("%s.h%d.O_full" % (wlname, bh), _pick(step.Of, B, H, T, bh, rows), Of, True)
        check_close("%s.h%d.O_sparse" % (wlname, bh), _pick(step.Os, B, H, T, bh, rows), Os, True)
        np.testing.assert_allclose(_pick(step.lse_f, B, H, T, bh, rows)[..., 0], lf, rtol=0, atol=2e-3)
        np.testing.assert_allclose(_pick(step.lse_s, B, H, T, bh, rows)[..., 0], ls, rtol=0, atol=2e-3)
        np.testing.assert_allclose(_pick(delta, B, H, T, bh, rows)[..., 0], ora.dropped_mass(ls, lf), rtol=0,
                                   atol=5e-3)
        if backward:
            # The main stream's backward with the seeded dO.  The other stream receives only the
            # alignment slope, |dL/do| <= max(w) / (B*H*T*d) ~ 1e-8 here, far below the tolerance,
            # so the oracle leaves it out.
            a = ora.attn_bwd(f["Q"], f["K"], f["V"], f["dO"], s, dims.scale, sel if main == "sparse" else None,
                             rows, rows)
            for nm, got, ref in zip(("dQ", "dK", "dV"), (step.dQ, step.dK, step.dV), a):
                check_close("%s.h%d.%s.%s" % (wlname, bh, main, nm), _pick(got, B, H, T, bh, rows), ref, False)
    return report


def test_prefill_8k():
    _run("prefill", 16, heads=[0, 15], n_rows=256, backward=False)


def test_train_4k():
    _run("train", 8, heads=[0, 63], n_rows=256, backward=True)


def test_long_32k():
    _run("long", 16, heads=[0], n_rows=192, backward=True, main="sparse")


def test_long_32k_full_stream_main():
    # the bench's other parity of step: the seeded dO goes to the full stream
    _run("long", 16, heads=[5], n_rows=128, backward=True, main="full")


@pytest.mark.parametrize("k", [4, 8, 16, 32, 64])
def test_sweep_128k(k):
    _run("sweep", k, heads=[3], n_rows=128, backward=False)

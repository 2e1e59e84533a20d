"""Rotary positions (ssa_rope) against the fp64 oracle: the rotation of Q and K
(bf16, query and key head counts, a position offset, scaling factors 1 and 4,
a large base), its transpose on fp32 gradients, and one whole step whose Q and K
carry rotary positions, against the oracle chain rotate -> path -> rotate back."""
import numpy as np
import pytest

import oracle as ora
from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import inputs, ops

from .helpers import bf16_half_ulp, check_close, check_gpu_selection, to_device, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from block_top_sparse_b200 import build
    build.build()
    ora.build()


@pytest.mark.parametrize("base,factor,pos0", [(10000.0, 1.0, 0), (500000.0, 4.0, 777)])
def test_rope_matches_oracle(base, factor, pos0):
    g = inputs.generate(inputs.WORKLOADS["long"], H=4, T=4096)
    dims = L.make_dims(1, 4, 4096, 128, 128, 1)
    Q = to_device(g["Q"], "bf16")
    ops.rope(dims, Q, pos0=pos0, base=base, factor=factor)
    ref = ora.rope(inputs.to_float64(g["Q"], "bf16").reshape(4, 4096, 128), pos0, base, factor)
    got = to_np(Q).reshape(4, 4096, 128)
    # one bf16 rounding of the rotated value, plus fp32 arithmetic
    assert np.all(np.abs(got - ref) <= bf16_half_ulp(ref) + 1e-5 * (np.abs(ref) + 1))
    # the transpose on fp32 data undoes it
    X = torch.from_numpy(ref.astype(np.float32)).reshape(1, 4, 4096, 128).cuda()
    ops.rope(dims, X, pos0=pos0, base=base, factor=factor, transpose=True)
    back = ora.rope(ref, pos0, base, factor, inverse=True)
    np.testing.assert_allclose(to_np(X).reshape(4, 4096, 128), back, rtol=0, atol=2e-5)
    assert L.ssa_get_device_error() == L.SSA_OK


@pytest.mark.parametrize("main", ["full", "sparse"])
def test_step_with_rotary_positions(main):
    base, factor, k = 500000.0, 4.0, 4
    g = inputs.group_kv(inputs.generate(inputs.WORKLOADS["long"], H=4, T=1024, with_dO=True), 2)
    w = g["wl"]
    dims = L.make_dims(1, 4, 1024, 128, 128, k, Hkv=2)
    dev = {key: to_device(g[key], "bf16") for key in ("Q", "K", "V", "dO")}
    step = ops.SSAStep(dims, main=main, grad_fp32=True, rope=(base, factor))
    step.forward(dev["Q"], dev["K"], dev["V"])
    step.main_grad_buffer().copy_(dev["dO"])
    step.backward(dev["Q"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert L.ssa_get_device_error() == L.SSA_OK
    f = {key: inputs.to_float64(g[key], "bf16").reshape(-1, 1024, 128) for key in ("Q", "K", "V", "dO")}
    # the oracle chain on the rotated inputs as the GPU stored them (bf16; the rotation itself is checked
    # against the oracle's above and here), then the rotation's transpose of the gradients
    Qr, Kr = to_np(step.Qr).reshape(4, 1024, 128), to_np(step.Kr).reshape(2, 1024, 128)
    for got, x in ((Qr, f["Q"]), (Kr, f["K"])):
        ref = ora.rope(x, 0, base, factor)
        assert np.all(np.abs(got - ref) <= bf16_half_ulp(ref) + 1e-5 * (np.abs(ref) + 1))
    Kbar = ora.block_pool(Kr, w.s)
    sel = step.idx.cpu().numpy().reshape(2, 1024, k)
    check_gpu_selection(ora, "rope.step." + main, sel, Qr, Kbar, w.s, k)
    Of, _ = ora.attn_fwd(Qr, Kr, f["V"], w.s, dims.scale)
    Os, _ = ora.attn_fwd(Qr, Kr, f["V"], w.s, dims.scale, sel)
    check_close("rope.step.Of", to_np(step.Of).reshape(4, 1024, 128), Of, True)
    check_close("rope.step.Os", to_np(step.Os).reshape(4, 1024, 128), Os, True)
    gf, gs = ora.align_bwd(Of, Os)
    dOf = f["dO"] + gf if main == "full" else gf
    dOs = f["dO"] + gs if main == "sparse" else gs
    a = ora.attn_bwd(Qr, Kr, f["V"], dOf, w.s, dims.scale)
    b = ora.attn_bwd(Qr, Kr, f["V"], dOs, w.s, dims.scale, sel)
    dQ = ora.rope(a[0] + b[0], 0, base, factor, inverse=True)
    dK = ora.rope(a[1] + b[1], 0, base, factor, inverse=True)
    check_close("rope.step.dQ", to_np(step.dQ).reshape(4, 1024, 128), dQ, True)
    check_close("rope.step.dK", to_np(step.dK).reshape(2, 1024, 128), dK, True)
    check_close("rope.step.dV", to_np(step.dV).reshape(2, 1024, 128), a[2] + b[2], True)

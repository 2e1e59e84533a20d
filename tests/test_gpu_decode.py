"""Sparse decoding with a key/value cache (ssa_sparse_decode) against the fp64
oracle: for each sequence the oracle runs the training-path definitions on a
query tensor that holds the new query at row L (its selection row, and its
attention row over the selected blocks' tokens up to L).  Cache lengths cover
the first token, a token inside a block, a token that completes a block (the
pooled-key cache gains that block's mean, and nothing else changes) and the
last slot of the cache; grouped query heads share the selection."""
import numpy as np
import pytest

import oracle as ora
from block_top_sparse_b200 import _lib as L
from block_top_sparse_b200 import inputs, ops

from .helpers import TIE_REL, check_close, selection_report, to_device, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from block_top_sparse_b200 import build
    build.build()
    ora.build()


# groups of 1, 2, 4, 8 and 16 query heads per key/value head; blocks of 128 and 64 keys; caches of 16, 32,
# 512 and 1024 blocks (the selection's warp search holds 8, 16 or 32 scores per lane)
@pytest.mark.parametrize("H,Hkv,s,k,T", [(2, 2, 128, 4, 2048), (4, 2, 128, 5, 2048), (8, 2, 64, 6, 2048),
                                         (16, 2, 64, 4, 2048), (16, 1, 128, 3, 2048), (2, 1, 64, 8, 32768),
                                         (2, 1, 64, 8, 65536)])
def test_decode_matches_oracle(H, Hkv, s, k, T):
    B, d = 4, 128
    lens = np.array([0, 700, T - 1, 3 * s - 1], dtype=np.int32)  # the last one completes block 2
    g = inputs.group_kv(inputs.generate(inputs.WORKLOADS["long"], B=B, H=H, T=T), Hkv)
    Kc, Vc = to_device(g["K"], "bf16"), to_device(g["V"], "bf16")
    qraw = inputs.random_tensor((B, H, d), "bf16", seed=21, std=d ** -0.25)
    q = to_device(qraw, "bf16")
    dims = L.make_dims(B, H, T, d, s, k, Hkv=Hkv)
    # pooled-key cache: every block pooled once, then the rows the call may write set to a marker
    Kbar = ops.block_pool(dims, Kc)
    # cache rows past each sequence's new token hold NaN on the device (a cache's unwritten rows may hold
    # anything): the current block's keys and values past L must not reach the output, not even with
    # weight 0; the oracle reads the clean rows up to L only
    Kc4, Vc4 = Kc.view(B, Hkv, T, d), Vc.view(B, Hkv, T, d)
    for b, Lb in enumerate(lens):
        Kc4[b, :, Lb + 1:] = float("nan")
        Vc4[b, :, Lb + 1:] = float("nan")
    marker = -7.0
    for b, Lb in enumerate(lens):
        Kbar[b, :, Lb // s] = marker
    Kbar_before = Kbar.clone()
    idx = torch.empty((B, Hkv, k), dtype=torch.int32, device="cuda")
    o = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    ws = ops._ws(dims, L.SSA_OP_DECODE, "cuda")
    L.ssa_sparse_decode(dims, torch.from_numpy(lens).cuda(), q, Kc, Vc, Kbar, idx, o, lse, ws)
    torch.cuda.synchronize()
    assert L.ssa_get_device_error() == L.SSA_OK

    K64 = inputs.to_float64(g["K"], "bf16").reshape(B, Hkv, T, d)
    V64 = inputs.to_float64(g["V"], "bf16").reshape(B, Hkv, T, d)
    q64 = inputs.to_float64(qraw, "bf16").reshape(B, H, d)
    for b, Lb in enumerate(lens):
        Qfull = np.zeros((H, T, d))
        Qfull[:, Lb] = q64[b]
        Kbar_ref = ora.block_pool(K64[b], s)
        idx_ref, r1, r2 = ora.block_select(Qfull, Kbar_ref, s, k)
        got = idx.cpu().numpy()[b][:, None, :]          # [Hkv, 1, k]
        rep = selection_report(got, idx_ref[:, Lb:Lb + 1], r1[:, Lb:Lb + 1], r2[:, Lb:Lb + 1])
        assert rep["mismatch"] == 0, (b, rep)
        sel = idx_ref.copy()
        sel[:, Lb] = got[:, 0]
        o_ref, lse_ref = ora.attn_fwd(Qfull, K64[b], V64[b], s, dims.scale, sel, rows=[Lb])
        check_close("decode.b%d.o" % b, to_np(o[b]).reshape(H, 1, d), o_ref, True)
        np.testing.assert_allclose(to_np(lse[b]).reshape(H, 1), lse_ref, rtol=0, atol=2e-3)
        # pooled-key cache: block L // s is written exactly when token L completes it
        bt = Lb // s
        row = Kbar[b, :, bt].cpu().numpy()
        if (Lb + 1) % s == 0:
            np.testing.assert_allclose(row, Kbar_ref[:, bt], rtol=2e-6, atol=1e-7)
        else:
            assert np.all(row == marker)
    others = torch.ones(Kbar.shape[:3], dtype=torch.bool)
    for b, Lb in enumerate(lens):
        others[b, :, Lb // s] = False
    assert torch.equal(Kbar.cpu()[others], Kbar_before.cpu()[others])


def test_decode_reports_a_cache_length_out_of_range():
    B, H, T, d, s, k = 1, 2, 512, 128, 128, 2
    dims = L.make_dims(B, H, T, d, s, k)
    z = torch.zeros((B, H, T, d), dtype=torch.bfloat16, device="cuda")
    Kbar = torch.zeros((B, H, T // s, d), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, H, k), dtype=torch.int32, device="cuda")
    o = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    ws = ops._ws(dims, L.SSA_OP_DECODE, "cuda")
    bad = torch.tensor([T], dtype=torch.int32, device="cuda")
    L.ssa_sparse_decode(dims, bad, z[:, :, 0], z, z, Kbar, idx, o, lse, ws)
    assert L.ssa_get_device_error() == L.SSA_ERR_BAD_INPUT
    assert L.ssa_get_device_error() == L.SSA_OK
    assert bool((idx == -1).all())

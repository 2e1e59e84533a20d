"""Pins for the fp64 oracle, checked against things other than itself.

Every oracle function is pinned here by at least one of: a hand-computed closed
form, a special case that reduces to a library routine (torch SDPA, autograd,
smooth_l1_loss, numpy reductions), brute force on tiny inputs written as a
different algorithm (dense masks and full sorts), an invariant that the pages'
definitions fix (sparse == full when every preceding block is selected, rows
normalised over the selected set, the dropped-mass identity and bound), or
finite differences.  The paper's pages print no worked numbers, so no pin comes
from them directly.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from block_top_sparse_b200 import inputs


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


# --------------------------------------------------------------------------- pooling

def test_pool_closed_form(ora):
    BH, T, d, s = 2, 24, 3, 4
    t = np.arange(T, dtype=np.float64)[None, :, None]
    c = np.arange(d, dtype=np.float64)[None, None, :]
    K = np.broadcast_to(t * (c + 1) + 10.0 * np.arange(BH)[:, None, None], (BH, T, d))
    Kbar = ora.block_pool(K, s)
    j = np.arange(T // s, dtype=np.float64)[None, :, None]
    expect = (c + 1) * (j * s + (s - 1) / 2.0) + 10.0 * np.arange(BH)[:, None, None]
    np.testing.assert_array_equal(Kbar, expect)


def test_pool_matches_numpy_mean(ora):
    K = _rand((3, 64, 5), 1)
    np.testing.assert_allclose(ora.block_pool(K, 8), K.reshape(3, 8, 8, 5).mean(axis=2), rtol=0, atol=1e-15)


# --------------------------------------------------------------------------- selection

def test_select_hand_example(ora):
    # d = 1, q = 1, s = 2, k = 2: Kbar = [0.5, 3, 1, 7] -> every query keeps its own
    # block plus the best strictly preceding block.
    K = np.array([0, 1, 3, 3, 1, 1, 7, 7], dtype=np.float64)[None, :, None]
    Q = np.ones((1, 8, 1))
    Kbar = ora.block_pool(K, 2)
    np.testing.assert_array_equal(Kbar[0, :, 0], [0.5, 3.0, 1.0, 7.0])
    idx, r1, r2 = ora.block_select(Q, Kbar, 2, 2)
    expect = [[0, -1], [0, -1], [0, 1], [0, 1], [1, 2], [1, 2], [1, 3], [1, 3]]
    np.testing.assert_array_equal(idx[0], expect)
    # (k-1)-th and k-th candidate scores: block 3 queries rank {3, 1, 0.5}.
    assert r1[0, 6] == 3.0 and r2[0, 6] == 1.0
    assert np.isnan(r1[0, 0]) and np.isnan(r2[0, 2])


def test_select_tie_goes_to_lowest_index(ora):
    # All preceding blocks score exactly the same: the lowest indices win.
    s, k, T = 4, 3, 32
    K = np.ones((1, T, 2))
    Q = np.ones((1, T, 2))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    for t in range(T):
        bt = t // s
        pre = list(range(min(k - 1, bt)))
        np.testing.assert_array_equal(idx[0, t], pre + [bt] + [-1] * (k - 1 - len(pre)))


def _brute_select(Q, K, s, k):
    """Dense scores of every query against every block mean, then a full lexicographic sort."""
    BH, T, d = Q.shape
    nb = T // s
    means = np.stack([K[:, j * s:(j + 1) * s].sum(axis=1) / s for j in range(nb)], axis=1)
    scores = np.einsum("btd,bjd->btj", Q, means)
    out = np.full((BH, T, k), -1, dtype=np.int32)
    for b in range(BH):
        for t in range(T):
            bt = t // s
            cand = np.arange(bt)
            order = np.lexsort((cand, -scores[b, t, :bt]))  # primary: score desc; secondary: index asc
            pick = sorted(list(cand[order[:k - 1]]) + [bt])
            out[b, t, :len(pick)] = pick
    return out


@pytest.mark.parametrize("s,k", [(4, 1), (4, 3), (8, 4), (4, 16)])
def test_select_brute_force(ora, s, k):
    Q = _rand((2, 64, 6), 2)
    K = _rand((2, 64, 6), 3)
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    np.testing.assert_array_equal(idx, _brute_select(Q, K, s, k))
    assert ora.check_selection(idx, s)


def test_select_scale_invariance(ora):
    Q = _rand((1, 128, 8), 4)
    K = _rand((1, 128, 8), 5)
    Kbar = ora.block_pool(K, 8)
    a, _, _ = ora.block_select(Q, Kbar, 8, 5)
    b, _, _ = ora.block_select(Q * 3.5, Kbar * 0.25, 8, 5)
    np.testing.assert_array_equal(a, b)


def test_block_scores_hand_example(ora):
    # the hand example above: q = 1, Kbar = [0.5, 3, 1, 7]; query 6 (block 3) scores blocks 0-2
    K = np.array([0, 1, 3, 3, 1, 1, 7, 7], dtype=np.float64)[None, :, None]
    Q = np.ones((1, 8, 1))
    sc = ora.block_scores(Q, ora.block_pool(K, 2), 2, [0, 0], [6, 1])
    np.testing.assert_array_equal(sc[0, :3], [0.5, 3.0, 1.0])
    assert np.isnan(sc[0, 3]) and np.all(np.isnan(sc[1]))  # not candidates: j >= b(t)


@pytest.mark.parametrize("s,k", [(4, 3), (8, 5)])
def test_block_scores_rank_to_the_brute_force_selection(ora, s, k):
    # Sorting a row's candidate scores (score desc, index asc) and keeping k-1 plus b(t) gives the
    # brute-force selection, and ranks k-1, k are the r_(k-1), r_(k) block_select reports.
    Q = _rand((2, 64, 6), 12)
    K = _rand((2, 64, 6), 13)
    Kbar = ora.block_pool(K, s)
    idx, r1, r2 = ora.block_select(Q, Kbar, s, k)
    brute = _brute_select(Q, K, s, k)
    bh, t = np.meshgrid(np.arange(2), np.arange(64), indexing="ij")
    sc = ora.block_scores(Q, Kbar, s, bh.ravel(), t.ravel())
    for i, (b, tt) in enumerate(zip(bh.ravel(), t.ravel())):
        bt = tt // s
        cand = np.arange(bt)
        order = cand[np.lexsort((cand, -sc[i, :bt]))]
        pick = sorted(list(order[:k - 1]) + [bt])
        np.testing.assert_array_equal(brute[b, tt, :len(pick)], pick)
        if bt >= k:
            assert sc[i, order[k - 2]] == r1[b, tt] and sc[i, order[k - 1]] == r2[b, tt]


def test_check_selection_rejects_bad_rows(ora):
    good = np.array([[[0, -1], [0, 1]]], dtype=np.int32)  # T=2, s=1
    assert ora.check_selection(good, 1)
    for bad in ([[[0, -1], [1, 0]]], [[[-1, 0], [0, 1]]], [[[0, -1], [0, -1]]], [[[0, 0], [0, 1]]]):
        assert not ora.check_selection(np.array(bad, dtype=np.int32), 1)


# --------------------------------------------------------------------------- attention forward

def _dense_mask(idx, T, s):
    """mask[b, t, u] = key u is attended by query t (sparse stream), brute force."""
    BH = idx.shape[0]
    m = np.zeros((BH, T, T), dtype=bool)
    for b in range(BH):
        for t in range(T):
            for j in idx[b, t]:
                if j >= 0:
                    m[b, t, j * s:(j + 1) * s] = True
    return m & np.tril(np.ones((T, T), dtype=bool))[None]


def _dense_attn(Q, K, V, mask, scale):
    x = np.einsum("btd,bud->btu", Q, K) * scale
    x = np.where(mask, x, -np.inf)
    m = x.max(axis=-1, keepdims=True)
    p = np.exp(x - m)
    l = p.sum(axis=-1, keepdims=True)
    return np.einsum("btu,bud->btd", p / l, V), (m + np.log(l))[..., 0]


@pytest.mark.parametrize("scale", [0.125, 1.0])
def test_full_fwd_matches_torch_sdpa(ora, scale):
    Q, K, V = (_rand((3, 40, 8), i) for i in (6, 7, 8))
    O, lse = ora.attn_fwd(Q, K, V, 4, scale)
    ref = F.scaled_dot_product_attention(torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V),
                                         is_causal=True, scale=scale).numpy()
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    x = torch.from_numpy(np.einsum("btd,bud->btu", Q, K) * scale)
    x = x.masked_fill(~torch.tril(torch.ones(40, 40, dtype=torch.bool)), -float("inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(x, dim=-1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("s,k", [(4, 1), (4, 3), (8, 2)])
def test_sparse_fwd_brute_force(ora, s, k):
    T = 64
    Q, K, V = (_rand((2, T, 6), i) for i in (9, 10, 11))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    O, lse = ora.attn_fwd(Q, K, V, s, 0.3, idx)
    Ob, lseb = _dense_attn(Q, K, V, _dense_mask(idx, T, s), 0.3)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lseb, rtol=0, atol=1e-12)


def test_sparse_equals_full_when_all_blocks_selected(ora):
    T, s = 48, 4
    Q, K, V = (_rand((2, T, 5), i) for i in (12, 13, 14))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, T // s)
    Os, ls = ora.attn_fwd(Q, K, V, s, 0.5, idx)
    Of, lf = ora.attn_fwd(Q, K, V, s, 0.5)
    np.testing.assert_array_equal(Os, Of)
    np.testing.assert_array_equal(ls, lf)
    # and row-wise for queries with fewer than k preceding blocks, at smaller k
    k = 4
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    Os, _ = ora.attn_fwd(Q, K, V, s, 0.5, idx)
    early = np.arange(T) // s < k
    np.testing.assert_array_equal(Os[:, early], Of[:, early])


def test_rows_normalised_over_selected_set(ora):
    T, s, k = 32, 4, 2
    Q, K = _rand((1, T, 4), 15), _rand((1, T, 4), 16)
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    O, _ = ora.attn_fwd(Q, K, np.ones((1, T, 4)), s, 1.0, idx)
    np.testing.assert_allclose(O, 1.0, rtol=0, atol=1e-14)
    # identical keys: uniform weights over S(t), so o_t is the plain mean of V over S(t)
    V = _rand((1, T, 4), 17)
    O, lse = ora.attn_fwd(Q, np.ones((1, T, 4)), V, s, 1.0, idx)
    mask = _dense_mask(idx, T, s)[0]
    for t in range(T):
        np.testing.assert_allclose(O[0, t], V[0, mask[t]].mean(axis=0), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, t], Q[0, t].sum() + np.log(mask[t].sum()), rtol=0, atol=1e-13)


def test_fwd_closed_form_two_tokens(ora):
    # d = 1, T = 2, s = 1: o_0 = v_0; o_1 = (e^{a} v_0 + e^{b} v_1)/(e^{a} + e^{b}) with a = c q1 k0, b = c q1 k1.
    q, kk, v, c = [0.3, -1.2], [0.7, 2.0], [1.5, -4.0], 0.9
    O, lse = ora.attn_fwd(np.array(q)[None, :, None], np.array(kk)[None, :, None], np.array(v)[None, :, None], 1, c)
    a, b = c * q[1] * kk[0], c * q[1] * kk[1]
    assert O[0, 0, 0] == pytest.approx(v[0], abs=1e-15)
    assert O[0, 1, 0] == pytest.approx((np.exp(a) * v[0] + np.exp(b) * v[1]) / (np.exp(a) + np.exp(b)), abs=1e-14)
    assert lse[0, 0] == pytest.approx(c * q[0] * kk[0], abs=1e-15)
    assert lse[0, 1] == pytest.approx(np.log(np.exp(a) + np.exp(b)), abs=1e-14)


def test_fwd_row_subset(ora):
    Q, K, V = (_rand((2, 32, 4), i) for i in (18, 19, 20))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, 4), 4, 3)
    O, lse = ora.attn_fwd(Q, K, V, 4, 0.5, idx)
    rows = [31, 0, 17]
    Or, lr = ora.attn_fwd(Q, K, V, 4, 0.5, idx, rows=rows)
    np.testing.assert_array_equal(Or, O[:, rows])
    np.testing.assert_array_equal(lr, lse[:, rows])


def test_dropped_mass_identity_and_bound(ora):
    # Appendix B reading: with full weights p_u and delta = sum_{u not in S} p_u,
    # o_f = (1 - delta) o_s + delta * u_drop, so |o_f - o_s| <= 2 delta max|v|.
    T, s, k = 64, 4, 3
    Q, K, V = (_rand((2, T, 6), i) for i in (21, 22, 23))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    Os, ls = ora.attn_fwd(Q, K, V, s, 0.7, idx)
    Of, lf = ora.attn_fwd(Q, K, V, s, 0.7)
    delta = ora.dropped_mass(ls, lf)
    x = np.einsum("btd,bud->btu", Q, K) * 0.7
    causal = np.tril(np.ones((T, T), dtype=bool))[None]
    p = np.where(causal, np.exp(x - x.max(axis=-1, keepdims=True)), 0.0)
    p /= p.sum(axis=-1, keepdims=True)
    drop = causal & ~_dense_mask(idx, T, s)
    np.testing.assert_allclose(delta, np.where(drop, p, 0).sum(-1), rtol=0, atol=1e-12)
    u_drop_times_delta = np.einsum("btu,bud->btd", np.where(drop, p, 0), V)
    np.testing.assert_allclose(Of, (1 - delta)[..., None] * Os + u_drop_times_delta, rtol=0, atol=1e-12)
    vmax = np.linalg.norm(V, axis=-1).max()
    assert np.all(np.linalg.norm(Of - Os, axis=-1) <= 2 * delta * vmax + 1e-12)
    assert np.all(delta[:, : k * s] == pytest.approx(0.0, abs=1e-14))


# --------------------------------------------------------------------------- attention backward

def _torch_grads(Q, K, V, dO, mask, scale):
    q, k, v = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    x = torch.einsum("btd,bud->btu", q, k) * scale
    x = x.masked_fill(~torch.from_numpy(mask), -float("inf"))
    o = torch.einsum("btu,bud->btd", torch.softmax(x, dim=-1), v)
    (o * torch.from_numpy(dO)).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


def test_full_bwd_matches_autograd_sdpa(ora):
    Q, K, V, dO = (_rand((2, 36, 5), i) for i in (24, 25, 26, 27))
    dQ, dK, dV = ora.attn_bwd(Q, K, V, dO, 4, 0.4)
    q, k, v = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=0.4)
    (o * torch.from_numpy(dO)).sum().backward()
    np.testing.assert_allclose(dQ, q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dK, k.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dV, v.grad.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("s,k", [(4, 2), (8, 3)])
def test_sparse_bwd_matches_autograd_dense_mask(ora, s, k):
    T = 64
    Q, K, V, dO = (_rand((2, T, 6), i) for i in (28, 29, 30, 31))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    dQ, dK, dV = ora.attn_bwd(Q, K, V, dO, s, 0.6, idx)
    gq, gk, gv = _torch_grads(Q, K, V, dO, _dense_mask(idx, T, s), 0.6)
    np.testing.assert_allclose(dQ, gq, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dK, gk, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dV, gv, rtol=0, atol=1e-12)


def test_sparse_bwd_finite_differences(ora):
    # Selection held fixed (no gradient through it): perturb Q/K/V with idx frozen.
    T, s, k, scale, eps = 24, 4, 2, 0.8, 1e-6
    Q, K, V, dO = (_rand((1, T, 3), i) for i in (32, 33, 34, 35))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    grads = ora.attn_bwd(Q, K, V, dO, s, scale, idx)
    rng = np.random.default_rng(36)
    for which in range(3):
        for _ in range(6):
            t, c = int(rng.integers(T)), int(rng.integers(3))
            args = [Q.copy(), K.copy(), V.copy()]
            args[which][0, t, c] += eps
            up = (ora.attn_fwd(*args, s, scale, idx)[0] * dO).sum()
            args[which][0, t, c] -= 2 * eps
            dn = (ora.attn_fwd(*args, s, scale, idx)[0] * dO).sum()
            assert grads[which][0, t, c] == pytest.approx((up - dn) / (2 * eps), rel=1e-6, abs=1e-8)


def test_dropped_keys_get_zero_gradient(ora):
    # Upstream gradient on one query row only: keys outside S(t) must get exactly 0.
    T, s, k = 64, 4, 2
    Q, K, V, dO = (_rand((1, T, 4), i) for i in (37, 38, 39, 40))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    mask = _dense_mask(idx, T, s)[0]
    for t in (63, 40, 17):
        g = np.zeros_like(dO)
        g[0, t] = dO[0, t]
        _, dK, dV = ora.attn_bwd(Q, K, V, g, s, 1.0, idx)
        assert (~mask[t]).sum() > 0
        assert np.all(dK[0, ~mask[t]] == 0) and np.all(dV[0, ~mask[t]] == 0)
        assert np.all(np.abs(dV[0, mask[t]]).sum(-1) > 0)


def test_bwd_row_subsets(ora):
    Q, K, V, dO = (_rand((2, 32, 4), i) for i in (41, 42, 43, 44))
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, 4), 4, 3)
    full = ora.attn_bwd(Q, K, V, dO, 4, 0.5, idx)
    qr, kr = [5, 31, 0], [31, 2, 16, 7]
    sub = ora.attn_bwd(Q, K, V, dO, 4, 0.5, idx, qrows=qr, krows=kr)
    np.testing.assert_allclose(sub[0], full[0][:, qr], rtol=0, atol=1e-14)
    np.testing.assert_allclose(sub[1], full[1][:, kr], rtol=0, atol=1e-14)
    np.testing.assert_allclose(sub[2], full[2][:, kr], rtol=0, atol=1e-14)


# --------------------------------------------------------------------------- grouped-query attention

def _grouped_inputs(G, BHk=2, T=64, d=6, seed=60):
    Q = _rand((BHk * G, T, d), seed)
    K = _rand((BHk, T, d), seed + 1)
    V = _rand((BHk, T, d), seed + 2)
    dO = _rand((BHk * G, T, d), seed + 3)
    return Q, K, V, dO


@pytest.mark.parametrize("G,s,k", [(2, 4, 3), (4, 8, 2), (3, 4, 16)])
def test_grouped_select_brute_force(ora, G, s, k):
    # a key head's selection ranks blocks by the sum of its G query heads' scores
    Q, K, _, _ = _grouped_inputs(G)
    Kbar = ora.block_pool(K, s)
    idx, _, _ = ora.block_select(Q, Kbar, s, k)
    BHk, T = K.shape[0], K.shape[1]
    means = np.stack([K[:, j * s:(j + 1) * s].mean(axis=1) for j in range(T // s)], axis=1)
    scores = np.einsum("gitd,gjd->gtj", Q.reshape(BHk, G, T, -1), means)
    for b in range(BHk):
        for t in range(T):
            bt = t // s
            cand = np.arange(bt)
            pick = sorted(list(cand[np.lexsort((cand, -scores[b, t, :bt]))][:k - 1]) + [bt])
            np.testing.assert_array_equal(idx[b, t, :len(pick)], pick)
    assert ora.check_selection(idx, s)


@pytest.mark.parametrize("G", [2, 4])
def test_grouped_full_attention_matches_sdpa_and_autograd(ora, G):
    # grouped-query attention is attention with each key/value head repeated for its G query heads
    Q, K, V, dO = _grouped_inputs(G)
    T, scale = Q.shape[1], 0.4
    mask = np.broadcast_to(np.tril(np.ones((T, T), dtype=bool)), (Q.shape[0], T, T))
    O, lse = ora.attn_fwd(Q, K, V, 4, scale)
    Kr, Vr = np.repeat(K, G, axis=0), np.repeat(V, G, axis=0)
    ref = F.scaled_dot_product_attention(torch.tensor(Q), torch.tensor(Kr), torch.tensor(Vr), is_causal=True,
                                         scale=scale).numpy()
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    dq, dk, dv = ora.attn_bwd(Q, K, V, dO, 4, scale)
    q, kk, vv = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    o = F.scaled_dot_product_attention(q, kk.repeat_interleave(G, dim=0), vv.repeat_interleave(G, dim=0),
                                       is_causal=True, scale=scale)
    (o * torch.from_numpy(dO)).sum().backward()
    for got, want in ((dq, q.grad), (dk, kk.grad), (dv, vv.grad)):
        np.testing.assert_allclose(got, want.numpy(), rtol=0, atol=1e-11)
    assert dk.shape == K.shape and dv.shape == V.shape


@pytest.mark.parametrize("G,s,k", [(2, 4, 2), (4, 8, 3)])
def test_grouped_sparse_attention_matches_dense_mask(ora, G, s, k):
    # every query head of a group attends over its key head's selection
    Q, K, V, dO = _grouped_inputs(G)
    T, scale = Q.shape[1], 0.7
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, s), s, k)
    mask = np.repeat(_dense_mask(idx, T, s), G, axis=0)
    Kr, Vr = np.repeat(K, G, axis=0), np.repeat(V, G, axis=0)
    O, lse = ora.attn_fwd(Q, K, V, s, scale, idx)
    O_ref, lse_ref = _dense_attn(Q, Kr, Vr, mask, scale)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)
    dq, dk, dv = ora.attn_bwd(Q, K, V, dO, s, scale, idx)
    q, kk, vv = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    x = torch.einsum("btd,bud->btu", q, kk.repeat_interleave(G, dim=0)) * scale
    x = x.masked_fill(~torch.from_numpy(mask), -float("inf"))
    o = torch.einsum("btu,bud->btd", torch.softmax(x, dim=-1), vv.repeat_interleave(G, dim=0))
    (o * torch.from_numpy(dO)).sum().backward()
    for got, want in ((dq, q.grad), (dk, kk.grad), (dv, vv.grad)):
        np.testing.assert_allclose(got, want.numpy(), rtol=0, atol=1e-11)


# --------------------------------------------------------------------------- rotary positions

def test_rope_two_dims_closed_form(ora):
    # d = 2: one pair turned by the position itself (base^0 = 1)
    X = np.array([[[1.0, 0.0], [0.6, -0.8], [2.0, 3.0]]])
    out = ora.rope(X, pos0=5)
    for t in range(3):
        a = 5.0 + t
        x0, x1 = X[0, t]
        np.testing.assert_allclose(out[0, t], [x0 * np.cos(a) - x1 * np.sin(a), x0 * np.sin(a) + x1 * np.cos(a)],
                                   rtol=0, atol=1e-15)


def test_rope_scores_depend_on_relative_position_only(ora):
    q = _rand((1, 1, 16), 70)
    k = _rand((1, 1, 16), 71)
    def score(tq, tk, factor=1.0):
        return float(ora.rope(q, pos0=tq, factor=factor).ravel() @ ora.rope(k, pos0=tk, factor=factor).ravel())
    for factor in (1.0, 4.0):
        assert score(100, 37, factor) == pytest.approx(score(1163, 1100, factor), rel=1e-9, abs=1e-12)


def test_rope_inverse_norm_and_scaling(ora):
    X = _rand((2, 32, 8), 72)
    Y = ora.rope(X, pos0=3, base=500000.0, factor=4.0)
    np.testing.assert_allclose(np.linalg.norm(Y, axis=-1), np.linalg.norm(X, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(ora.rope(Y, pos0=3, base=500000.0, factor=4.0, inverse=True), X, rtol=0, atol=1e-13)
    # factor 4 at position 4m is the plain rotation at position m
    Z = ora.rope(X[:, ::4], pos0=0, base=500000.0)
    np.testing.assert_allclose(ora.rope(X, pos0=0, base=500000.0, factor=4.0)[:, ::4], Z, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- alignment loss

@pytest.mark.parametrize("beta,ws,wc", [(1.0, 1.0, 1.0), (0.5, 0.3, 2.0)])
def test_align_matches_torch(ora, beta, ws, wc):
    Of, Os = _rand((2, 3, 7, 5), 45), _rand((2, 3, 7, 5), 46)
    of, os_ = torch.tensor(Of, requires_grad=True), torch.tensor(Os, requires_grad=True)
    L = ws * F.smooth_l1_loss(of, os_.detach(), beta=beta) + wc * F.smooth_l1_loss(os_, of.detach(), beta=beta)
    (1.7 * L).backward()
    assert ora.align_fwd(Of, Os, beta, ws, wc) == pytest.approx(L.item(), rel=1e-14)
    gf, gs = ora.align_bwd(Of, Os, beta, ws, wc, 1.7)
    np.testing.assert_allclose(gf, of.grad.numpy(), rtol=0, atol=1e-16)
    np.testing.assert_allclose(gs, os_.grad.numpy(), rtol=0, atol=1e-16)


def test_align_stop_gradient_symmetry(ora):
    Of, Os = _rand((4, 9), 47), _rand((4, 9), 48)
    gf, gs = ora.align_bwd(Of, Os, 1.0, 1.0, 1.0, 1.0)
    np.testing.assert_array_equal(gs, -gf)
    gf, gs = ora.align_bwd(Of, Os, 1.0, 1.0, 0.0, 1.0)   # one-way: commitment off
    assert np.all(gs == 0) and np.any(gf != 0)


def test_align_finite_differences(ora):
    Of, Os = _rand((3, 4), 49), _rand((3, 4), 50) * 0.3
    ws, wc, eps = 0.7, 1.3, 1e-7
    # Each direction's gradient is the finite difference of its own term with the
    # other stream held constant (stop-gradient).
    gf, gs = ora.align_bwd(Of, Os, 1.0, ws, wc, 1.0)
    for i in range(3):
        for j in range(4):
            a, b = Of.copy(), Of.copy()
            a[i, j] += eps
            b[i, j] -= eps
            fd = (ora.align_fwd(a, Os, 1.0, ws, 0.0) - ora.align_fwd(b, Os, 1.0, ws, 0.0)) / (2 * eps)
            assert gf[i, j] == pytest.approx(fd, rel=1e-5, abs=1e-9)
            a, b = Os.copy(), Os.copy()
            a[i, j] += eps
            b[i, j] -= eps
            fd = (ora.align_fwd(Of, a, 1.0, 0.0, wc) - ora.align_fwd(Of, b, 1.0, 0.0, wc)) / (2 * eps)
            assert gs[i, j] == pytest.approx(fd, rel=1e-5, abs=1e-9)


@pytest.mark.parametrize("beta,ws,wc", [(1.0, 1.0, 1.0), (0.5, 0.3, 2.0)])
def test_align_l2_matches_torch_mse(ora, beta, ws, wc):
    # adjusted L2 (section 7.5): 0.5 x^2 / beta for every x = mse_loss / (2 beta), both directions
    Of, Os = _rand((2, 3, 7, 5), 51) * 2.0, _rand((2, 3, 7, 5), 52)
    of, os_ = torch.tensor(Of, requires_grad=True), torch.tensor(Os, requires_grad=True)
    L = (ws * F.mse_loss(of, os_.detach()) + wc * F.mse_loss(os_, of.detach())) / (2 * beta)
    (1.3 * L).backward()
    assert ora.align_fwd(Of, Os, beta, ws, wc, kind="l2") == pytest.approx(L.item(), rel=1e-14)
    gf, gs = ora.align_bwd(Of, Os, beta, ws, wc, 1.3, kind="l2")
    np.testing.assert_allclose(gf, of.grad.numpy(), rtol=1e-14, atol=1e-18)
    np.testing.assert_allclose(gs, os_.grad.numpy(), rtol=1e-14, atol=1e-18)


def test_align_l2_equals_smooth_l1_inside_beta(ora):
    # the two kinds agree where every |o_f - o_s| < beta, and L2 exceeds SmoothL1 beyond it
    Of = _rand((6, 8), 53) * 0.1
    Os = Of + _rand((6, 8), 54) * 0.1
    assert ora.align_fwd(Of, Os, 2.0, 1.0, 1.0, kind="l2") == pytest.approx(ora.align_fwd(Of, Os, 2.0, 1.0, 1.0),
                                                                            rel=1e-14)
    far = Os + 5.0
    assert ora.align_fwd(Of, far, 1.0, 1.0, 1.0, kind="l2") > ora.align_fwd(Of, far, 1.0, 1.0, 1.0)


# --------------------------------------------------------------------------- input generator

def test_bf16_rounding_is_rne():
    u = 2.0 ** -7  # bf16 spacing on [1, 2)
    x = np.array([1.0, 1 + u / 2, 1 + 3 * u / 2, 1 + u / 4, 1 + 3 * u / 4, -2.5, 0.0], dtype=np.float32)
    back = inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(x))
    # ties go to the even mantissa: 1 + u/2 -> 1, 1 + 3u/2 -> 1 + 2u
    expect = np.array([1.0, 1.0, 1 + 2 * u, 1.0, 1 + u, -2.5, 0.0], dtype=np.float32)
    np.testing.assert_array_equal(back, expect)


def test_generator_shapes_and_determinism():
    wl = inputs.WORKLOADS["prefill"]
    a = inputs.generate(wl, T=512, H=2)
    b = inputs.generate(wl, T=512, H=2)
    for key in ("Q", "K", "V"):
        assert a[key].shape == (1, 2, 512, 128) and a[key].dtype == np.uint16
        np.testing.assert_array_equal(a[key], b[key])
    assert "dO" not in a
    t = inputs.generate(inputs.WORKLOADS["tiny"])
    assert t["Q"].dtype == np.float32 and t["dO"].shape == (1, 2, 1024, 64)
    std = inputs.to_float64(a["Q"], "bf16").std()
    assert 0.8 * 128 ** -0.25 < std < 1.2 * 128 ** -0.25


def test_planted_blocks_are_found(ora):
    # Queries are planted toward 4 preceding blocks; the oracle's selection at k=16
    # should contain most of them for queries with many preceding blocks.
    wl = inputs.WORKLOADS["prefill"]
    g = inputs.generate(wl, T=2048, H=1)
    Q = inputs.to_float64(g["Q"], "bf16")[0]
    K = inputs.to_float64(g["K"], "bf16")[0]
    idx, _, _ = ora.block_select(Q, ora.block_pool(K, wl.s), wl.s, 5)
    # with k-1 = 4 picks among >= 16 candidates, a planted structure makes the
    # selection far from uniform: its blocks have clearly higher mean scores.
    Kbar = ora.block_pool(K, wl.s)
    sc = np.einsum("td,jd->tj", Q[0], Kbar[0])
    t = np.arange(1024, 2048)
    bt = t // wl.s
    chosen = np.take_along_axis(sc[t], np.clip(idx[0, t, :4], 0, None), axis=1).mean()
    pool_mean = np.array([sc[tt, :b].mean() for tt, b in zip(t, bt)]).mean()
    pool_std = np.array([sc[tt, :b].std() for tt, b in zip(t, bt)]).mean()
    assert chosen > pool_mean + 1.5 * pool_std


def test_bwd_with_stored_bf16_output_matches_dense_formulas(ora):
    # The backward given the forward's output as stored in bfloat16: D_t = dO_t . bf16(o_t), the rest of the
    # gradient formulas unchanged.  Dense numpy formulas with torch's bfloat16 rounding as the pin.
    T, d, s, scale = 16, 4, 4, 0.5
    Q, K, V, dO = (_rand((1, T, d), i) for i in (40, 41, 42, 43))
    q, k, v, g = Q[0], K[0], V[0], dO[0]
    S = scale * q @ k.T
    S[np.triu_indices(T, 1)] = -np.inf
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    o_b = torch.from_numpy(P @ v).to(torch.bfloat16).double().numpy()
    D = (g * o_b).sum(axis=1, keepdims=True)
    dS = P * (g @ v.T - D)
    want = (scale * dS @ k, scale * dS.T @ q, P.T @ g)
    got = ora.attn_bwd(Q, K, V, dO, s, scale, stored_o="bf16")
    exact = ora.attn_bwd(Q, K, V, dO, s, scale)
    for gg, w in zip(got, want):
        np.testing.assert_allclose(gg[0], w, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[2], exact[2], rtol=0, atol=1e-12)  # dV does not involve D
    assert np.abs(got[0] - exact[0]).max() > 0  # the rounding is visible in dQ


def test_oracle_regression_against_committed_golden(ora):
    # tests/golden/tiny_case.json: the oracle's outputs on a tiny seeded case, written by make_golden.py
    import json
    import os
    import importlib.util
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(here, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    doc = json.load(open(os.path.join(here, "tiny_case.json")))
    x = {k: np.array(v) for k, v in doc["inputs"].items()}
    for k, v in mg.inputs().items():
        np.testing.assert_array_equal(x[k], v)  # the generator still produces the stored inputs
    got = mg.compute(x)
    for k, v in doc["outputs"].items():
        np.testing.assert_allclose(np.asarray(got[k], dtype=np.float64), np.array(v, dtype=np.float64),
                                   rtol=1e-12, atol=1e-12, err_msg=k)

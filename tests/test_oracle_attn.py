"""Pins of the oracle's block-sparse attention (NABLA page, 手法: NABLA,
"拡張": attention is computed on the kept blocks; 問題提起: full attention is
the all-pairs O((T H W)^2) case).  Library routines fix the expected values:
torch's float64 scaled_dot_product_attention (dense, and with the block mask
expanded to an additive -inf token mask), torch.autograd for the gradients,
and central finite differences of the oracle's own forward."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

L = 64


def _rand_problem(BH=2, nb=6, D=32, seed=0):
    rng = np.random.default_rng(seed)
    N = nb * L
    q, k, v, do = (rng.standard_normal((BH, N, D)) for _ in range(4))
    return q, k, v, do


def _random_lists(BH, nb, density, seed):
    rng = np.random.default_rng(seed)
    dense = rng.random((BH, nb, nb)) < density
    dense |= np.eye(nb, dtype=bool)[None]
    return _lists(dense)


def _lists(dense):
    BH, nb, _ = dense.shape
    row_idx = np.zeros((BH, nb, nb), np.uint16)
    row_cnt = np.zeros((BH, nb), np.int32)
    col_idx = np.zeros((BH, nb, nb), np.uint16)
    col_cnt = np.zeros((BH, nb), np.int32)
    for b in range(BH):
        for i in range(nb):
            j = np.flatnonzero(dense[b, i])
            row_idx[b, i, :j.size] = j
            row_cnt[b, i] = j.size
            c = np.flatnonzero(dense[b, :, i])
            col_idx[b, i, :c.size] = c
            col_cnt[b, i] = c.size
    return dense, row_idx, row_cnt, col_idx, col_cnt


def _sdpa(q, k, v, dense, scale):
    tq, tk, tv = (torch.tensor(a) for a in (q, k, v))
    tok = torch.tensor(dense).repeat_interleave(L, 1).repeat_interleave(L, 2)
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=tok, scale=scale)
    logits = scale * tq @ tk.transpose(1, 2)
    lse = torch.logsumexp(logits.masked_fill(~tok, float("-inf")), dim=-1)
    return o.numpy(), lse.numpy()


def test_dense_limit_equals_sdpa(oracle_mod):
    q, k, v, _ = _rand_problem()
    BH, N, D = q.shape
    nb = N // L
    dense, ri, rc, _, _ = _lists(np.ones((BH, nb, nb), bool))
    scale = 1 / np.sqrt(D)
    o, lse = oracle_mod.attn_fwd(q, k, v, ri, rc, scale)
    tq, tk, tv = (torch.tensor(a) for a in (q, k, v))
    want = F.scaled_dot_product_attention(tq, tk, tv, scale=scale).numpy()
    assert np.max(np.abs(o.reshape(BH, N, D) - want)) < 1e-12
    wl = torch.logsumexp(scale * tq @ tk.transpose(1, 2), -1).numpy()
    assert np.max(np.abs(lse.reshape(BH, N) - wl)) < 1e-12


def test_block_diagonal_is_per_block_attention(oracle_mod):
    q, k, v, _ = _rand_problem(seed=1)
    BH, N, D = q.shape
    nb = N // L
    dense, ri, rc, _, _ = _lists(np.broadcast_to(np.eye(nb, dtype=bool), (BH, nb, nb)).copy())
    scale = 0.3
    o, _ = oracle_mod.attn_fwd(q, k, v, ri, rc, scale)
    blk = lambda a: torch.tensor(a).reshape(BH * nb, L, D)
    want = F.scaled_dot_product_attention(blk(q), blk(k), blk(v), scale=scale)
    assert np.max(np.abs(o.reshape(-1) - want.numpy().reshape(-1))) < 1e-12


@pytest.mark.parametrize("density", [0.2, 0.5])
def test_sparse_equals_masked_dense(oracle_mod, density):
    q, k, v, _ = _rand_problem(seed=2)
    BH, N, D = q.shape
    nb = N // L
    dense, ri, rc, _, _ = _random_lists(BH, nb, density, seed=3)
    scale = 1 / np.sqrt(D)
    o, lse = oracle_mod.attn_fwd(q, k, v, ri, rc, scale)
    wo, wl = _sdpa(q, k, v, dense, scale)
    assert np.max(np.abs(o.reshape(BH, N, D) - wo)) < 1e-12
    assert np.max(np.abs(lse.reshape(BH, N) - wl)) < 1e-12
    # a selection returns exactly the corresponding rows
    sel = [(1, 3), (0, 0), (1, nb - 1)]
    so, sl = oracle_mod.attn_fwd(q, k, v, ri, rc, scale, sel=sel)
    for s, (b, i) in enumerate(sel):
        assert np.array_equal(so[s], o.reshape(BH, nb, L, D)[b, i])
        assert np.array_equal(sl[s], lse.reshape(BH, nb, L)[b, i])


def test_backward_equals_autograd(oracle_mod):
    q, k, v, do = _rand_problem(seed=4)
    BH, N, D = q.shape
    nb = N // L
    dense, ri, rc, ci, cc = _random_lists(BH, nb, 0.4, seed=5)
    scale = 1 / np.sqrt(D)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, ri, rc, ci, cc, scale)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    tok = torch.tensor(dense).repeat_interleave(L, 1).repeat_interleave(L, 2)
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=tok, scale=scale)
    o.backward(torch.tensor(do))
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.max(np.abs(got.reshape(BH, N, D) - t.grad.numpy())) < 1e-10
    # selections
    sdq, sdk, sdv = oracle_mod.attn_bwd(q, k, v, do, ri, rc, ci, cc, scale,
                                        dq_sel=[(1, 2)], kv_sel=[(0, 4), (1, 0)])
    assert np.array_equal(sdq[0], dq.reshape(BH, nb, L, D)[1, 2])
    assert np.array_equal(sdk[1], dk.reshape(BH, nb, L, D)[1, 0])
    assert np.array_equal(sdv[0], dv.reshape(BH, nb, L, D)[0, 4])


def test_backward_matches_finite_differences(oracle_mod):
    q, k, v, g = _rand_problem(BH=1, nb=3, D=8, seed=6)
    BH, N, D = q.shape
    nb = N // L
    dense, ri, rc, ci, cc = _random_lists(BH, nb, 0.5, seed=7)
    scale = 0.4

    def loss(q_, k_, v_):
        o, _ = oracle_mod.attn_fwd(q_, k_, v_, ri, rc, scale)
        return float(np.sum(o.reshape(BH, N, D) * g))

    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, g, ri, rc, ci, cc, scale)
    rng = np.random.default_rng(8)
    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for _ in range(4):
            n, d = int(rng.integers(N)), int(rng.integers(D))
            args = [q.copy(), k.copy(), v.copy()]
            args[which][0, n, d] += h
            up = loss(*args)
            args[which][0, n, d] -= 2 * h
            dn = loss(*args)
            fd = (up - dn) / (2 * h)
            assert abs(fd - grad.reshape(BH, N, D)[0, n, d]) < 1e-6 * max(1.0, abs(fd))

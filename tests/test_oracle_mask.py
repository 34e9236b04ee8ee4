"""Pins of the oracle's whole mask: pooled map -> CDF cut -> OR with the STA
window and the diagonal -> compact row lists, bit rows and column lists
(NABLA page, 手法: NABLA: "拡張" and "STA とのハイブリッド統合", M = M_∇ ∨ M_STA).
The float64 definition is checked against an independent numpy restatement
(library matmul + stable argsort); the decision-precision mask is checked
against the float64 one away from the cut's rounding band."""
import numpy as np
import pytest
import torch

from adaptive_block_sparse_fractal_b200 import synth


def _inputs(oracle_mod, w, seed0=0):
    inp = synth.make_inputs(w, seed0)
    out = {}
    for name in ("q", "k"):
        raw = synth.bits(inp[name]).reshape(w.BH, w.N, w.D)
        out[name] = oracle_mod.flatten_tokens(raw, w.T, w.H, w.W, w.P)
    return out


def _numpy_mask_f64(qbar, kbar, grid, p, scale, window):
    """Independent restatement with library routines."""
    BH, nb, D = qbar.shape
    T, Hp, Wp = grid
    s = scale * np.einsum("bid,bjd->bij", qbar, kbar)
    prob = np.exp(s - s.max(axis=2, keepdims=True))
    prob /= prob.sum(axis=2, keepdims=True)
    keep = np.zeros_like(prob, dtype=bool)
    for bh in range(BH):
        for i in range(nb):
            if p >= 1:
                keep[bh, i] = True
                continue
            order = np.lexsort((np.arange(nb), -s[bh, i]))  # score desc, index asc
            cum = np.cumsum(prob[bh, i, order])
            before = np.concatenate([[0.0], cum[:-1]])
            keep[bh, i, order[before < p]] = True
    idx = np.arange(nb)
    t, h, ww = idx // (Hp * Wp), (idx // Wp) % Hp, idx % Wp
    sta = ((np.abs(t[:, None] - t[None, :]) <= window[0] // 2)
           & (np.abs(h[:, None] - h[None, :]) <= window[1] // 2)
           & (np.abs(ww[:, None] - ww[None, :]) <= window[2] // 2))
    return keep | sta[None] | np.eye(nb, dtype=bool)[None]


def _check_structure(m, dense):
    BH, nb = m["row_cnt"].shape
    for bh in range(BH):
        for i in range(nb):
            c = m["row_cnt"][bh, i]
            lst = m["row_idx"][bh, i, :c]
            assert np.all(np.diff(lst.astype(np.int64)) > 0)
            assert np.array_equal(lst, np.flatnonzero(dense[bh, i]))
            bits = np.unpackbits(m["bits"][bh, i].view(np.uint8), bitorder="little")[:nb]
            assert np.array_equal(bits.astype(bool), dense[bh, i])
        if "col_idx" in m:
            for j in range(nb):
                c = m["col_cnt"][bh, j]
                assert np.array_equal(m["col_idx"][bh, j, :c], np.flatnonzero(dense[bh, :, j]))


@pytest.mark.parametrize("wname,p", [("tiny", 0.9), ("tiny", 0.5), ("tiny", 1.0)])
def test_f64_mask_matches_numpy_restatement(oracle_mod, wname, p):
    w = synth.WORKLOADS[wname]
    x = _inputs(oracle_mod, w)
    qb, kb = oracle_mod.pool_f64(x["q"]), oracle_mod.pool_f64(x["k"])
    m = oracle_mod.mask_f64(qb, kb, w.grid_blocks, p, w.scale, w.window)
    want = _numpy_mask_f64(qb, kb, w.grid_blocks, p, w.scale, w.window)
    dense = oracle_mod.lists_to_dense(m["row_idx"], m["row_cnt"])
    assert np.array_equal(dense, want)
    _check_structure(m, dense)


def _band(m64, p, eps):
    return (np.abs(m64["cum_before"] - p) < eps) | (np.abs(m64["cum_at"] - p) < eps)


@pytest.mark.parametrize("p", [0.5, 0.8, 0.95])
def test_decision_precision_mask_matches_f64_outside_band(oracle_mod, p):
    # a reduced Small-like problem: 4 heads, 8 x 32 x 32 latent (128 blocks)
    w = synth.Workload("s4", 1, 4, 8, 32, 32, 128, (2, 4, 4), p)
    x = _inputs(oracle_mod, w)
    m32 = oracle_mod.build_mask(x["q"], x["k"], w.grid_blocks, p, w.scale, w.window)
    m64 = oracle_mod.mask_f64(oracle_mod.pool_f64(x["q"]), oracle_mod.pool_f64(x["k"]),
                              w.grid_blocks, p, w.scale, w.window)
    d32 = oracle_mod.lists_to_dense(m32["row_idx"], m32["row_cnt"])
    d64 = oracle_mod.lists_to_dense(m64["row_idx"], m64["row_cnt"])
    band = _band(m64, p, 1e-5)
    assert band.mean() < 0.01
    assert np.array_equal(d32[~band], d64[~band])
    _check_structure(m32, d32)


def test_mask_invariants(oracle_mod):
    w = synth.WORKLOADS["tiny"]
    x = _inputs(oracle_mod, w)
    qb, kb = oracle_mod.pool_f32(x["q"]), oracle_mod.pool_f32(x["k"])
    nb = w.nb
    # p = 0 without STA leaves exactly the diagonal
    m = oracle_mod.mask(qb, kb, w.grid_blocks, 0.0, w.scale, w.window, oracle_mod.NO_STA)
    d = oracle_mod.lists_to_dense(m["row_idx"], m["row_cnt"])
    assert np.array_equal(d, np.broadcast_to(np.eye(nb, dtype=bool), d.shape))
    # p = 0 with STA leaves STA | diagonal
    m0 = oracle_mod.mask(qb, kb, w.grid_blocks, 0.0, w.scale, w.window)
    d0 = oracle_mod.lists_to_dense(m0["row_idx"], m0["row_cnt"])
    T, Hp, Wp = w.grid_blocks
    for i in range(nb):
        for j in range(nb):
            assert d0[0, i, j] == oracle_mod.sta(i, j, Hp, Wp, w.window)
    # p = 1 keeps every block; the full window alone also does
    m1 = oracle_mod.mask(qb, kb, w.grid_blocks, 1.0, w.scale, w.window, oracle_mod.NO_STA)
    assert np.all(m1["row_cnt"] == nb)
    mf = oracle_mod.mask(qb, kb, w.grid_blocks, 0.0, w.scale, w.window, oracle_mod.FULL_STA)
    assert np.all(mf["row_cnt"] == nb)
    # the adaptive part grows with p and every kept set contains STA | diag
    prev = d0
    for p in (0.3, 0.6, 0.9, 0.99):
        mp = oracle_mod.mask(qb, kb, w.grid_blocks, p, w.scale, w.window)
        dp = oracle_mod.lists_to_dense(mp["row_idx"], mp["row_cnt"])
        assert np.all(prev <= dp)
        prev = dp

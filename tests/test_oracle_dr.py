"""Pins of the oracle's DynamicRad-style masks ("DynamicRad: Content-Adaptive
Sparse Attention for Long Video Diffusion", section 2.A "Dual-Mode Strategy"):

Static-Ratio (no content scoring, a retention ratio by temporal distance):
  - the number of blocks kept per (row, frame) equals the closed form
    k(dt) = ceil(min(1, max(lambda, gamma^dt)) * Hp * Wp), evaluated here in
    exact rational arithmetic for parameters whose powers are exact in binary;
  - the kept patches of a frame are the nearest to the query's patch, checked
    by brute force against every dropped patch (distance, then index);
  - gamma = 1 or lambda = 1 keep everything; a vanishing gamma keeps the
    query's own frame and the nearest patch of the adjacent frames only.
Dynamic-Threshold (pre-softmax logits as the importance proxy, a threshold):
  - tau = 0 keeps exactly the row's top-scoring blocks, tau = inf all of them;
  - the kept set grows with tau;
  - the rule restated with numpy float32 arithmetic on the oracle's (pinned)
    scores; and a block is kept iff its softmax weight is at least e^-tau of
    the best one's, on every block not within rounding of that boundary."""
from fractions import Fraction

import numpy as np
import pytest

from adaptive_block_sparse_fractal_b200 import synth


def _frame_counts(m, grid):
    T, Hp, Wp = grid
    HW = Hp * Wp
    BH, nb = m["row_cnt"].shape
    out = np.zeros((BH, nb, T), dtype=np.int64)
    for bh in range(BH):
        for i in range(nb):
            lst = m["row_idx"][bh, i, :m["row_cnt"][bh, i]].astype(np.int64)
            np.add.at(out[bh, i], lst // HW, 1)
    return out


@pytest.mark.parametrize("grid,gamma,lam", [((6, 3, 4), 0.75, 0.0), ((5, 4, 4), 0.5, 0.125),
                                            ((8, 2, 3), 0.875, 0.25)])
def test_static_counts_follow_the_closed_form(oracle_mod, grid, gamma, lam):
    T, Hp, Wp = grid
    HW = Hp * Wp
    m = oracle_mod.dr_static(2, grid, gamma, lam, flags=oracle_mod.NO_STA)
    counts = _frame_counts(m, grid)
    g, l_ = Fraction(gamma), Fraction(lam)
    for i in range(T * HW):
        ti = i // HW
        for t in range(T):
            dt = abs(t - ti)
            r = min(Fraction(1), max(l_, g ** dt))
            k = -((-r * HW) // 1)  # ceil, exactly
            want = k + (1 if (t == ti and k == 0) else 0)  # the diagonal is always kept
            assert counts[0, i, t] == want and counts[1, i, t] == want, (i, t)


def test_static_keeps_the_nearest_patches(oracle_mod):
    grid = (4, 4, 5)
    T, Hp, Wp = grid
    HW = Hp * Wp
    m = oracle_mod.dr_static(1, grid, 0.6, 0.05, flags=oracle_mod.NO_STA)
    dense = oracle_mod.lists_to_dense(m["row_idx"], m["row_cnt"])[0]
    for i in range(T * HW):
        qh, qw = (i % HW) // Wp, i % Wp
        for t in range(T):
            key = [((p // Wp - qh) ** 2 + (p % Wp - qw) ** 2, p) for p in range(HW)]
            kept = [key[p] for p in range(HW) if dense[i, t * HW + p]]
            dropped = [key[p] for p in range(HW) if not dense[i, t * HW + p]]
            if kept and dropped:
                assert max(kept) < min(dropped), (i, t)


def test_static_special_cases(oracle_mod):
    grid = (5, 3, 3)
    nb = 45
    assert np.all(oracle_mod.dr_static(1, grid, 1.0, 0.0, flags=oracle_mod.NO_STA)["row_cnt"] == nb)
    assert np.all(oracle_mod.dr_static(1, grid, 0.3, 1.0, flags=oracle_mod.NO_STA)["row_cnt"] == nb)
    # a vanishing gamma: the query's frame whole (dt = 0 has ratio 1), the one
    # nearest patch of each adjacent frame (ceil of a positive ratio: the
    # query's own patch), nothing farther (gamma^2 underflows to 0)
    m = oracle_mod.dr_static(1, grid, 1e-300, 0.0, flags=oracle_mod.NO_STA)
    counts = _frame_counts(m, grid)[0]
    dense = oracle_mod.lists_to_dense(m["row_idx"], m["row_cnt"])[0]
    for i in range(nb):
        ti = i // 9
        want = [9 if t == ti else (1 if abs(t - ti) == 1 else 0) for t in range(5)]
        assert list(counts[i]) == want
        for t in (ti - 1, ti + 1):
            if 0 <= t < 5:
                assert dense[i, t * 9 + i % 9]
    # with the STA window the union also holds the 3x3x3 neighbourhood
    ms = oracle_mod.dr_static(1, grid, 1e-300, 0.0)
    d = oracle_mod.lists_to_dense(ms["row_idx"], ms["row_cnt"])[0]
    for i in range(nb):
        for j in range(nb):
            if oracle_mod.sta(i, j, 3, 3, (3, 3, 3)):
                assert d[i, j]


def _pooled(oracle_mod, w, seed=0):
    inp = synth.make_inputs(w, seed)
    x = {n: oracle_mod.flatten_tokens(synth.bits(inp[n]).reshape(w.BH, w.N, w.D), w.T, w.H, w.W,
                                      w.P) for n in ("q", "k")}
    return oracle_mod.pool_f32(x["q"]), oracle_mod.pool_f32(x["k"])


def test_threshold_extremes_and_monotonicity(oracle_mod):
    w = synth.WORKLOADS["tiny"]
    qb, kb = _pooled(oracle_mod, w)
    s = oracle_mod.scores_f32(qb, kb, w.scale)
    m0 = oracle_mod.dr_threshold(qb, kb, w.grid_blocks, 0.0, w.scale, flags=oracle_mod.NO_STA)
    top = s == s.max(axis=2, keepdims=True)
    d0 = oracle_mod.lists_to_dense(m0["row_idx"], m0["row_cnt"])
    assert np.array_equal(d0, top | np.eye(w.nb, dtype=bool)[None])
    mi = oracle_mod.dr_threshold(qb, kb, w.grid_blocks, np.inf, w.scale, flags=oracle_mod.NO_STA)
    assert np.all(mi["row_cnt"] == w.nb)
    prev = d0
    for tau in (0.1, 0.5, 1.0, 2.0, 5.0):
        m = oracle_mod.dr_threshold(qb, kb, w.grid_blocks, tau, w.scale)
        d = oracle_mod.lists_to_dense(m["row_idx"], m["row_cnt"])
        assert np.all(prev <= d)
        prev = d


@pytest.mark.parametrize("wname,tau", [("tiny", 0.3), ("tiny", 0.7),
                                       ("small4", 0.4), ("small4", 1.5)])
def test_threshold_matches_numpy_and_softmax_ratio(oracle_mod, wname, tau):
    w = (synth.WORKLOADS["tiny"] if wname == "tiny"
         else synth.Workload("small4", 1, 4, 8, 32, 32, 128, (2, 4, 4), 0.8))
    qb, kb = _pooled(oracle_mod, w)
    s = oracle_mod.scores_f32(qb, kb, w.scale)
    m = oracle_mod.dr_threshold(qb, kb, w.grid_blocks, tau, w.scale, flags=oracle_mod.NO_STA)
    got = np.zeros(s.shape, dtype=bool)
    for bh in range(w.BH):
        for i in range(w.nb):
            sel = m["row_idx"][bh, i, :m["row_cnt"][bh, i]]
            got[bh, i, sel] = True
    # numpy float32 restatement
    smax = s.max(axis=2, keepdims=True)
    keep = (smax - s) <= np.float32(tau)
    assert keep.dtype == bool
    want = keep | np.eye(w.nb, dtype=bool)[None]
    assert np.array_equal(got, want)
    # softmax weights relative to the row's best, in float64, off the boundary
    ratio = np.exp(s.astype(np.float64) - smax.astype(np.float64))
    clear = np.abs(np.log(ratio) + tau) > 1e-5
    assert np.array_equal((ratio >= np.exp(-tau))[clear] | np.eye(w.nb, dtype=bool)[None]
                          .repeat(w.BH, 0)[clear], want[clear])
    assert 0 < keep.mean() < 1

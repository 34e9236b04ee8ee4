"""Pins of the oracle's pooled block scores in decision precision (NABLA page,
手法: NABLA, bullet "縮小されたアテンション": the attention map over the pooled
blocks), s_ij = (float32 fused multiply-add chain over d ascending of
qbar_i[d] * kbar_j[d]) * scale, and of the mask built from given scores.

Each pin is fixed by arithmetic worked out by hand or by an exact integer
product, not by re-running the oracle's own formula:
  - small-integer pooled means make every partial sum exact, so the scores
    equal the integer matrix product times a power-of-two scale;
  - hand-made rows whose value depends on the summation order, on whether
    products are fused, and on which operand is the query;
  - random means against the float64 product within the float32 error bound
    of a length-D chain;
  - the mask from the scores equals the mask from the pooled means."""
import numpy as np
import pytest

from adaptive_block_sparse_fractal_b200 import synth


def _scores(oracle_mod, q_rows, k_rows, scale):
    q = np.asarray(q_rows, dtype=np.float32)[None]
    k = np.asarray(k_rows, dtype=np.float32)[None]
    return oracle_mod.scores_f32(q, k, scale)[0]


def test_integer_means_equal_exact_integer_product(oracle_mod):
    rng = np.random.default_rng(3)
    BH, nb, D = 2, 9, 128
    q = rng.integers(-8, 9, size=(BH, nb, D))
    k = rng.integers(-8, 9, size=(BH, nb, D))
    # every partial sum is an integer below 2^24: the chain is exact
    want = np.einsum("bid,bjd->bij", q, k) * 0.125  # int64, then an exact scale
    got = oracle_mod.scores_f32(q.astype(np.float32), k.astype(np.float32), 0.125)
    assert got.dtype == np.float32
    assert np.array_equal(got.astype(np.float64), want.astype(np.float64))
    # rows follow the query, columns the key: the transpose differs
    assert not np.array_equal(got, np.swapaxes(got, 1, 2))


def test_summation_order_is_ascending(oracle_mod):
    # Two rows with the same three products, k = (1, 1, 1), worked by hand:
    #   q = (2^25, 1, -2^25): 2^25; 2^25 + 1 rounds to 2^25 (float32 spacing 4
    #     there); then 0.  A float64 accumulator would give 1.
    #   q = (2^25, -2^25, 1): 2^25; 0; then 1.  Run in descending order,
    #     1 - 2^25 is a tie between -2^25 and -2^25 + 2 (spacing 2), rounded to
    #     the even -2^25, and the chain ends at 0.
    got = _scores(oracle_mod, [[2.0 ** 25, 1.0, -(2.0 ** 25)], [2.0 ** 25, -(2.0 ** 25), 1.0]],
                  [[1.0, 1.0, 1.0]], 1.0)
    assert got[0, 0] == 0.0
    assert got[1, 0] == 1.0


def test_products_are_fused(oracle_mod):
    # q = (-1, 1 + 2^-12), k = (1, 1 + 2^-12): after -1 the chain adds
    # (1 + 2^-12)^2 = 1 + 2^-11 + 2^-24 in one rounding, giving 2^-11 + 2^-24
    # exactly.  Rounding the product first (a tie, to even: 1 + 2^-11) would
    # give 2^-11.
    a = 1.0 + 2.0 ** -12
    got = _scores(oracle_mod, [[-1.0, a]], [[1.0, a]], 1.0)
    assert got[0, 0] == np.float32(2.0 ** -11 + 2.0 ** -24)
    assert got[0, 0] != np.float32(2.0 ** -11)


def test_scale_is_applied_after_the_chain_in_float32(oracle_mod):
    # s = 3 exactly; 3 * 0.1f rounds once in float32
    got = _scores(oracle_mod, [[1.0, 2.0]], [[1.0, 1.0]], 0.1)
    assert got[0, 0] == np.float32(3.0) * np.float32(0.1)


def test_random_means_within_float32_chain_bound(oracle_mod):
    rng = np.random.default_rng(7)
    BH, nb, D = 3, 17, 128
    q = rng.standard_normal((BH, nb, D)).astype(np.float32)
    k = rng.standard_normal((BH, nb, D)).astype(np.float32)
    scale = np.float32(1.0 / np.sqrt(D))
    got = oracle_mod.scores_f32(q, k, scale).astype(np.float64)
    exact = np.einsum("bid,bjd->bij", q.astype(np.float64), k.astype(np.float64))
    mag = np.einsum("bid,bjd->bij", np.abs(q.astype(np.float64)), np.abs(k.astype(np.float64)))
    u = 2.0 ** -24
    bound = (D * u * mag + u * np.abs(exact)) * float(scale) * 1.01
    assert np.all(np.abs(got - exact * float(scale)) <= bound + 1e-30)
    # a dropped term, a transposed operand or a missing scale fails the bound
    assert np.abs(got - exact * float(scale)).max() < 1e-4
    assert not np.allclose(got, np.swapaxes(got, 1, 2), atol=1e-3)


@pytest.mark.parametrize("p", [0.3, 0.7, 0.95])
def test_mask_from_scores_equals_mask_from_means(oracle_mod, p):
    w = synth.Workload("s2", 1, 2, 4, 32, 32, 64, (2, 4, 4), p)
    inp = synth.make_inputs(w, 0)
    x = {n: oracle_mod.flatten_tokens(synth.bits(inp[n]).reshape(w.BH, w.N, w.D),
                                      w.T, w.H, w.W, w.P) for n in ("q", "k")}
    qb, kb = oracle_mod.pool_f32(x["q"]), oracle_mod.pool_f32(x["k"])
    m = oracle_mod.mask(qb, kb, w.grid_blocks, p, w.scale, w.window)
    s = oracle_mod.scores_f32(qb, kb, w.scale)
    ms = oracle_mod.mask_from_scores(s, w.grid_blocks, p, w.window)
    for key in ("bits", "row_cnt", "col_cnt", "adapt_cnt"):
        assert np.array_equal(m[key], ms[key]), key
    assert np.array_equal(m["margin"], ms["margin"])
    # and each row's adaptive set is the cut of that row alone
    for bh in range(w.BH):
        for i in range(0, w.nb, 13):
            keep = oracle_mod.cut_row_fixed(s[bh, i], p)
            assert keep.sum() == ms["adapt_cnt"][bh, i]

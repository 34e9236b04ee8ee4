"""Pins of the oracle's per-row CDF cut (NABLA page, 手法: NABLA, bullets
"縮小されたアテンション" and "CDF 閾値処理": a full softmax map over the pooled
blocks; per row, the blocks whose cumulative probability exceeds 1 - thr are
kept).  Reading: p := thr; the kept set is the shortest prefix of the blocks in
descending probability (equal scores: lower index first) whose mass reaches
p; p >= 1 keeps everything."""
import itertools

import numpy as np
import pytest


def _softmax(s):
    e = np.exp(s - s.max())
    return e / e.sum()


def _brute_force_min_sets(prob, p):
    """All subsets (as bit masks) of minimum size whose mass reaches p."""
    nb = prob.size
    masks = np.arange(1 << nb, dtype=np.int64)
    member = ((masks[:, None] >> np.arange(nb)[None, :]) & 1).astype(np.float64)
    mass = member @ prob
    size = member.sum(axis=1)
    ok = mass >= p
    kmin = size[ok].min()
    return masks[ok & (size == kmin)], mass, kmin


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("p", [0.3, 0.7, 0.9, 0.99])
def test_brute_force_minimal_prefix_nb16(oracle_mod, seed, p):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(16) * (0.5 + seed)
    prob = _softmax(s)
    keep = oracle_mod.cut_row_f64(s, p)
    sets, mass, kmin = _brute_force_min_sets(prob, p)
    kept_mask = int(sum(1 << j for j in np.flatnonzero(keep)))
    assert keep.sum() == kmin  # no smaller subset reaches p
    assert kept_mask in set(sets.tolist())  # and the prefix is one of them
    # it is the heaviest of the minimum-size sets (the top-k set)
    assert np.isclose(mass[kept_mask], mass[sets].max(), rtol=0, atol=1e-15)


@pytest.mark.parametrize("seed", range(8))
def test_page_wording_ascending_cdf_exceeds_one_minus_p(oracle_mod, seed):
    # The page states the rule on the CDF: keep blocks whose cumulative
    # probability exceeds 1 - thr.  Accumulating in ascending order, block j's
    # CDF value is the mass of all blocks not above it (itself included).
    rng = np.random.default_rng(100 + seed)
    s = rng.standard_normal(40) * 2
    prob = _softmax(s)
    for p in (0.2, 0.5, 0.8, 0.95):
        order = np.argsort(prob, kind="stable")
        cdf = np.empty_like(prob)
        cdf[order] = np.cumsum(prob[order])
        want = cdf > 1.0 - p
        got = oracle_mod.cut_row_f64(s, p)
        # no ties in random data; skip values within rounding of the cut
        if np.min(np.abs(cdf - (1.0 - p))) < 1e-12:
            continue
        assert np.array_equal(got, want)


def test_special_values_and_ties(oracle_mod):
    s = np.array([0.1, 2.0, 2.0, -1.0, 0.5])
    for cut in (oracle_mod.cut_row_f64, oracle_mod.cut_row_fixed):
        assert not cut(s, 0.0).any()  # p = 0: empty adaptive set
        assert cut(s, 1.0).all()  # p = 1: every block
        k = cut(s, 1e-6)  # smallest p: the best block; tie -> lower index
        assert k.tolist() == [False, True, False, False, False]
        k = cut(s, 0.5)
        assert k.tolist() == [False, True, True, False, False]


@pytest.mark.parametrize("seed", range(4))
def test_monotone_in_p(oracle_mod, seed):
    rng = np.random.default_rng(200 + seed)
    s = rng.standard_normal(64) * 1.5
    ps = np.linspace(0, 1, 41)
    for cut in (oracle_mod.cut_row_f64, oracle_mod.cut_row_fixed):
        prev = cut(s, ps[0])
        for p in ps[1:]:
            cur = cut(s, p)
            assert np.all(prev <= cur)
            prev = cur


@pytest.mark.parametrize("seed", range(20))
def test_fixed_point_cut_matches_float64_definition(oracle_mod, seed):
    # The decision-precision cut (float32 scores, float64 weights, 2^-40
    # fixed-point mass) agrees with the float64 definition wherever the
    # float64 decision is not within 1e-9 of the threshold.
    rng = np.random.default_rng(300 + seed)
    nb = int(rng.integers(2, 300))
    s = (rng.standard_normal(nb) * rng.uniform(0.1, 4)).astype(np.float32)
    prob = _softmax(s.astype(np.float64))
    srt = np.sort(prob)[::-1]
    cum = np.concatenate([[0.0], np.cumsum(srt)])
    for p in (0.1, 0.5, 0.7, 0.9, 0.999):
        if np.min(np.abs(cum - p)) < 1e-9:
            continue
        assert np.array_equal(oracle_mod.cut_row_fixed(s, p),
                              oracle_mod.cut_row_f64(s.astype(np.float64), p))


def test_fixed_point_mass_is_exact_integer_arithmetic(oracle_mod):
    # Two blocks whose weights are exactly 1 and 2^-40: with p just above the
    # first block's share the second block is needed; the integer masses
    # make this decision exact.
    s = np.array([0.0, -40 * np.log(2.0)], dtype=np.float32)
    w1 = np.exp(np.float64(s[1]))  # ~2^-40
    share = 1.0 / (1.0 + w1)
    keep_lo = oracle_mod.cut_row_fixed(s, np.float32(0.5))
    assert keep_lo.tolist() == [True, False]
    # p = 1 - tiny still below the first block's share: nothing else kept
    assert share > np.float32(0.99999994)
    assert oracle_mod.cut_row_fixed(s, np.float32(0.99999994)).tolist() == [True, False]

"""Pins of the oracle's Sliding-Tile window (NABLA page, 手法: NABLA, section
"STA とのハイブリッド統合": the final mask is the OR of the adaptive mask and a
static STA window; the lay summary describes STA as attending the tile one
stands on and its immediate neighbours).  Reading: window (wt, wh, wv) in
blocks, centred, truncated at the grid border."""
import itertools

import numpy as np
import pytest


def _neighbours(i, grid, window):
    # independent restatement: enumerate offsets, drop those off the grid
    T, Hp, Wp = grid
    t, r = divmod(i, Hp * Wp)
    h, w = divmod(r, Wp)
    out = set()
    rt, rh, rw = (x // 2 for x in window)
    for dt, dh, dw in itertools.product(range(-rt, rt + 1), range(-rh, rh + 1),
                                        range(-rw, rw + 1)):
        tt, hh, ww = t + dt, h + dh, w + dw
        if 0 <= tt < T and 0 <= hh < Hp and 0 <= ww < Wp:
            out.add((tt * Hp + hh) * Wp + ww)
    return out


@pytest.mark.parametrize("window", [(3, 3, 3), (1, 3, 5), (5, 1, 3), (1, 1, 1)])
@pytest.mark.parametrize("grid", [(4, 2, 2), (5, 6, 7), (3, 4, 10)])
def test_window_matches_enumeration(oracle_mod, window, grid):
    T, Hp, Wp = grid
    nb = T * Hp * Wp
    for i in range(nb):
        got = {j for j in range(nb) if oracle_mod.sta(i, j, Hp, Wp, window)}
        assert got == _neighbours(i, grid, window)
        assert i in got


def test_interior_count_closed_form(oracle_mod):
    T, Hp, Wp = 7, 7, 9
    for window in [(3, 3, 3), (1, 3, 5), (5, 5, 3)]:
        i = ((T // 2) * Hp + Hp // 2) * Wp + Wp // 2
        cnt = sum(oracle_mod.sta(i, j, Hp, Wp, window) for j in range(T * Hp * Wp))
        assert cnt == window[0] * window[1] * window[2]
    # a corner block sees a 2 x 2 x 2 cube of a 3 x 3 x 3 window
    assert sum(oracle_mod.sta(0, j, Hp, Wp, (3, 3, 3)) for j in range(T * Hp * Wp)) == 8


def test_flags(oracle_mod):
    Hp, Wp, nb = 3, 4, 24
    for i, j in itertools.product(range(nb), repeat=2):
        assert oracle_mod.sta(i, j, Hp, Wp, (3, 3, 3), oracle_mod.FULL_STA)
        assert not oracle_mod.sta(i, j, Hp, Wp, (3, 3, 3), oracle_mod.NO_STA)
        assert oracle_mod.sta(i, j, Hp, Wp, (3, 3, 3)) == oracle_mod.sta(j, i, Hp, Wp, (3, 3, 3))

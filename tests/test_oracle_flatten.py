"""Pins of the oracle's fractal flattening (NABLA page, section 手法: NABLA,
"トークン再順序付け (Fractal Flattening)"): a hand-derived golden order, and the
properties the page fixes -- a bijection, P x P patches contiguous, time order
kept -- plus the inverse round trip."""
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden_cases():
    cases = []
    with open(os.path.join(HERE, "golden", "flatten_small_grids.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, order = line.split(":")
            T, H, W, P = (int(x) for x in head.split())
            cases.append((T, H, W, P, [int(x) for x in order.split()]))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: "T%dH%dW%dP%d" % c[:4])
def test_golden_order(oracle_mod, case):
    T, H, W, P, order = case
    perm = oracle_mod.permutation(T, H, W, P)  # perm[grid] = flat
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    assert inv.tolist() == order


GRIDS = [(4, 16, 16, 8), (3, 16, 24, 8), (2, 8, 8, 4), (1, 48, 80, 8)]


@pytest.mark.parametrize("grid", GRIDS)
def test_bijection_contiguity_time_order(oracle_mod, grid):
    T, H, W, P = grid
    perm = oracle_mod.permutation(T, H, W, P)
    N = T * H * W
    assert np.array_equal(np.sort(perm), np.arange(N))  # bijection
    inv = np.empty_like(perm)
    inv[perm] = np.arange(N)
    t = inv // (H * W)
    y = (inv // W) % H
    x = inv % W
    # time order kept: frame index never decreases along the flattened order
    assert np.all(np.diff(t) >= 0)
    # every aligned run of P*P flattened tokens is exactly one P x P patch
    L = P * P
    pt, py, px = t.reshape(-1, L), (y // P).reshape(-1, L), (x // P).reshape(-1, L)
    for a in (pt, py, px):
        assert np.all(a == a[:, :1])
    iy, ix = (y % P).reshape(-1, L), (x % P).reshape(-1, L)
    assert np.all(iy * P + ix == np.arange(L)[None, :])  # row-major inside
    # blocks are numbered (t, ph, pw) row-major
    blk = (pt[:, 0] * (H // P) + py[:, 0]) * (W // P) + px[:, 0]
    assert np.array_equal(blk, np.arange(N // L))


@pytest.mark.parametrize("inner", [2, 16, 256])
def test_round_trip_random_bytes(oracle_mod, inner):
    T, H, W, P = 2, 16, 24, 8
    rng = np.random.default_rng(7)
    x = rng.integers(0, 256, size=(3, T * H * W, inner), dtype=np.uint8)
    f = oracle_mod.flatten(x, T, H, W, P)
    assert not np.array_equal(f, x)
    back = oracle_mod.flatten(f, T, H, W, P, inverse=True)
    assert np.array_equal(back, x)
    # forward flatten moves grid token g to flat position perm[g]
    perm = oracle_mod.permutation(T, H, W, P)
    assert np.array_equal(f[:, perm], x)

"""nabla_build_mask on the GPU vs the oracle's decision-precision mask:
bit rows, row lists and column lists bit-exact (rows whose cut lies within
rounding of the threshold are counted; none are expected), pooled means
bit-exact, across p, STA flags, D, and ragged block counts."""
import numpy as np
import pytest
import torch

import oracle
from adaptive_block_sparse_fractal_b200 import nabla, synth

from gpu_util import Case, check_mask, to_np

pytestmark = pytest.mark.gpu

ODD = [
    synth.Workload("odd9", 1, 3, 3, 8, 24, 64, (1, 4, 4), 0.8),        # nb = 9 < one tile
    synth.Workload("odd130", 2, 2, 5, 16, 104, 128, (2, 4, 4), 0.7),   # nb = 130: ragged tile
    synth.Workload("odd1", 1, 1, 1, 8, 8, 128, (1, 8, 8), 0.5),        # a single block
    synth.Workload("odd150", 1, 2, 3, 40, 80, 64, (3, 8, 8), 0.9),     # nb = 150, D = 64
]


@pytest.fixture(scope="module")
def tiny():
    return Case(synth.WORKLOADS["tiny"], backward=True)


@pytest.fixture(scope="module")
def small():
    return Case(synth.WORKLOADS["small"])


@pytest.mark.parametrize("p", [0.0, 0.3, 0.7, 0.9, 0.999, 1.0])
@pytest.mark.parametrize("flags", [0, nabla.NO_STA, nabla.FULL_STA])
def test_tiny_mask(tiny, p, flags):
    gm = to_np(tiny.gpu_mask(p, flags))
    om = tiny.oracle_mask(p, flags)
    assert check_mask(gm, om) == 0


@pytest.mark.parametrize("p", [0.5, 0.8, 0.95])
def test_small_mask(small, p):
    gm = to_np(small.gpu_mask(p))
    om = small.oracle_mask(p)
    assert check_mask(gm, om) == 0


@pytest.mark.parametrize("w", ODD, ids=lambda w: w.name)
def test_ragged_shapes(w):
    c = Case(w)
    for p in (0.4, w.p, 1.0):
        assert check_mask(to_np(c.gpu_mask(p)), c.oracle_mask(p)) == 0


def _pooled_offset(w):
    """Byte offset of the pooled Q in a mask workspace: after the 256-byte
    status region and the front end's task counters (1 + B*heads ints)."""
    return 256 + (4 * (1 + w.BH) + 255) // 256 * 256


def test_pooled_means_bit_exact(small):
    w = small.w
    ws = nabla.workspace(small.shape, nabla.OP_BUILD_MASK, "cuda")
    nabla.build_mask(small.shape, small.params(), small.gpu["q"], small.gpu["k"], ws=ws)
    torch.cuda.synchronize()
    n = w.BH * w.nb * w.D
    raw = ws.cpu().numpy()
    base = _pooled_offset(w)
    qbar = raw[base:base + 4 * n].view(np.float32).reshape(w.BH, w.nb, w.D)
    off = base + ((4 * n + 255) // 256) * 256
    nbp = (w.nb + 3) // 4 * 4  # row stride of the transposed pooled K
    kbar_t = raw[off:off + 4 * w.BH * w.D * nbp].view(np.float32).reshape(w.BH, w.D, nbp)
    assert np.array_equal(qbar, oracle.pool_f32(small.cpu["q"]))
    assert np.array_equal(kbar_t[:, :, :w.nb].transpose(0, 2, 1), oracle.pool_f32(small.cpu["k"]))
    assert nabla.status(ws) == nabla.OK


def test_deterministic(small):
    a = to_np(small.gpu_mask())
    b = to_np(small.gpu_mask())
    for k in a:
        assert np.array_equal(a[k], b[k]), k


# Masks that do not depend on the scores (p <= 0, p >= 1, FULL_STA) take a
# path with neither pooling nor scores; windows other than 3x3x3 and patch
# grids narrower and wider than a warp exercise its block-coordinate stepping.
SCORE_FREE = [
    synth.Workload("win531_w5", 1, 2, 6, 24, 40, 64, (1, 4, 4), 0.7, window=(5, 3, 1)),     # Wp = 5
    synth.Workload("win173_w40", 1, 1, 3, 16, 320, 64, (1, 4, 4), 0.7, window=(1, 7, 3)),   # Wp = 40
    synth.Workload("win999", 1, 1, 4, 32, 32, 128, (2, 4, 4), 0.7, window=(9, 9, 9)),       # window > grid
]


@pytest.mark.parametrize("w", SCORE_FREE, ids=lambda w: w.name)
@pytest.mark.parametrize("p,flags", [(0.0, 0), (0.0, nabla.NO_STA), (1.0, 0), (0.5, nabla.FULL_STA),
                                     (0.6, 0)])
def test_score_free_paths_and_windows(w, p, flags):
    c = Case(w)
    gm = to_np(c.gpu_mask(p, flags))
    om = c.oracle_mask(p, flags)
    assert check_mask(gm, om) == 0
    if p >= 1.0 or flags & nabla.FULL_STA:
        assert np.all(gm["row_cnt"] == w.nb)
    if p == 0.0 and flags & nabla.NO_STA:
        assert np.all(gm["row_cnt"] == 1)  # the diagonal alone


GRID = [synth.WORKLOADS["small"], ODD[1], ODD[3], SCORE_FREE[1]]


@pytest.mark.parametrize("w", GRID, ids=lambda w: w.name)
@pytest.mark.parametrize("p,flags", [(None, 0), (0.0, 0), (0.5, nabla.FULL_STA)])
def test_build_mask_from_grid_matches_flatten_then_build(w, p, flags):
    """nabla_build_mask_grid: flattened copies bit-identical to the oracle's
    flattening, pooled means bit-identical to the oracle's pooling, and the
    mask identical to the one built from the separately flattened tensors."""
    c = Case(w)
    inp = synth.make_inputs(w, 0, with_dout=False)
    qg = inp["q"].reshape(w.BH, w.N, w.D).cuda()
    kg = inp["k"].reshape(w.BH, w.N, w.D).cuda()
    prm = c.params(p, flags)
    ws = nabla.workspace(c.shape, nabla.OP_BUILD_MASK, "cuda")
    qf, kf, gm = nabla.build_mask_grid(c.shape, prm, qg, kg, ws=ws)
    torch.cuda.synchronize()
    assert nabla.status(ws) == nabla.OK
    assert np.array_equal(synth.bits(qf.cpu()), c.cpu["q"])
    assert np.array_equal(synth.bits(kf.cpu()), c.cpu["k"])
    ref = to_np(c.gpu_mask(p, flags))
    got = to_np(gm)
    for key in ref:
        if key in ("row_idx", "col_idx"):
            cnt = ref["row_cnt" if key == "row_idx" else "col_cnt"]
            valid = np.arange(w.nb)[None, None, :] < cnt[..., None]
            assert np.array_equal(np.where(valid, got[key], 0), np.where(valid, ref[key], 0)), key
        else:
            assert np.array_equal(got[key], ref[key]), key
    assert check_mask(got, c.oracle_mask(p, flags)) == 0
    if p is None:  # the scored path pooled from the grid layout
        n = w.BH * w.nb * w.D
        raw = ws.cpu().numpy()
        base = _pooled_offset(w)
        qbar = raw[base:base + 4 * n].view(np.float32).reshape(w.BH, w.nb, w.D)
        assert np.array_equal(qbar, oracle.pool_f32(c.cpu["q"]))


# --------------------------------------------------------------------------
# NABLA_DEBUG_SCORES: the score phase checked on its own.  The kernel's float32
# scores must equal the oracle's score routine bit for bit, and the oracle's
# cut (and STA, diagonal) applied to the kernel's own scores must give the
# kernel's mask on every row.
# --------------------------------------------------------------------------
def _check_debug_scores(c, p, flags=0):
    prm = c.params(p, flags | nabla.DEBUG_SCORES)
    gm = to_np(nabla.build_mask(c.shape, prm, c.gpu["q"], c.gpu["k"]))
    qb, kb = oracle.pool_f32(c.cpu["q"]), oracle.pool_f32(c.cpu["k"])
    assert np.array_equal(gm["scores"], oracle.scores_f32(qb, kb, c.w.scale)), "scores differ"
    om = oracle.mask_from_scores(gm["scores"], c.w.grid_blocks, p, c.w.window, flags)
    assert check_mask(gm, om) == 0


@pytest.mark.parametrize("p", [0.5, 0.8, 0.95])
def test_debug_scores_small(small, p):
    _check_debug_scores(small, p)


@pytest.mark.parametrize("w", ODD, ids=lambda w: w.name)
def test_debug_scores_ragged(w):
    _check_debug_scores(Case(w), 0.6, nabla.NO_STA)


# --------------------------------------------------------------------------
# Tied scores.  The kernel ranks exactly only the histogram bucket that holds
# the last kept block; its blocks are held in shared memory when there are at
# most 256 of them and re-derived from the scores otherwise.  Key blocks built
# from a few repeated patterns make whole groups of blocks tie, so both forms
# run, and the ties are broken by block index as the definition says.
# --------------------------------------------------------------------------
def _repeat_k_blocks(w, patterns):
    def mutate(inp):
        B, h, T, H, W, D = inp["k"].shape
        g = torch.Generator().manual_seed(11)
        V = torch.randn(B, h, patterns, D, generator=g).to(torch.bfloat16)
        t = torch.arange(T)[:, None, None]
        y = torch.arange(H)[None, :, None]
        x = torch.arange(W)[None, None, :]
        blk = (t * (H // 8) + y // 8) * (W // 8) + x // 8           # [T, H, W]
        inp["k"] = V[:, :, blk % patterns].contiguous()              # [B, h, T, H, W, D]
    return mutate


TIES = [
    (synth.Workload("ties1_nb128", 1, 2, 8, 32, 32, 128, (2, 4, 4), 0.7), 1),     # every score equal
    (synth.Workload("ties5_nb1200", 1, 2, 20, 48, 80, 128, (2, 8, 8), 0.7), 5),   # 240 per group
    (synth.Workload("ties3_nb2048", 1, 1, 32, 64, 64, 128, (2, 8, 8), 0.6), 3),   # > 256 per group
    (synth.Workload("ties1_nb600", 1, 1, 10, 48, 80, 64, (2, 8, 8), 0.45), 1),    # D = 64
]


@pytest.mark.parametrize("w,patterns", TIES, ids=lambda x: getattr(x, "name", str(x)))
def test_tied_scores(w, patterns):
    c = Case(w, mutate=_repeat_k_blocks(w, patterns))
    for p in (0.2, w.p, 0.97):
        gm = to_np(c.gpu_mask(p))
        om = c.oracle_mask(p)
        assert check_mask(gm, om) == 0
        _check_debug_scores(c, p)


def test_front_end_wait_timeout_is_reported_and_the_context_survives():
    # nabla_build_mask_grid runs the pooling and the scores in one persistent
    # launch whose score tiles wait (bounded) for their head's pooling.  The
    # test aid makes every such wait expect one tile too many with a 1 ms
    # limit: the status must read NABLA_ERR_TIMEOUT, and the next call on the
    # same context and workspace must be correct.
    w = GRID[1]
    c = Case(w)
    inp = synth.make_inputs(w, 0, with_dout=False)
    qg = inp["q"].reshape(w.BH, w.N, w.D).cuda()
    kg = inp["k"].reshape(w.BH, w.N, w.D).cuda()
    ws = nabla.workspace(c.shape, nabla.OP_BUILD_MASK, "cuda")
    nabla.build_mask_grid(c.shape, c.params(flags=nabla.DEBUG_TIMEOUT), qg, kg, ws=ws)
    assert nabla.status(ws) == nabla.ERR_TIMEOUT
    _, _, gm = nabla.build_mask_grid(c.shape, c.params(), qg, kg, ws=ws)
    assert nabla.status(ws) == nabla.OK
    assert check_mask(to_np(gm), c.oracle_mask()) == 0

"""Full-size parity on the benchmark's workloads, in the launch configuration
bench.py times: the 720p-like shape (76,800 tokens, 40 heads, 1,200 blocks)
with its training backward, and the long clip (92,160 tokens, 12 heads,
1,440 blocks) over its p sweep.

Masks: every row, bit-exact against the oracle.  Attention: seeded samples of
query blocks (forward, dQ) and key blocks (dK, dV) that the float64 oracle
computes exactly, within max-abs 2e-2 / mean-abs 2e-3."""
import numpy as np
import pytest
import torch

import oracle
from adaptive_block_sparse_fractal_b200 import nabla, synth

from gpu_util import Case, assert_close, bf16_to_f64, check_mask, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

L = 64


@pytest.fixture(scope="module")
def train720():
    return Case(synth.WORKLOADS["train"])


@pytest.fixture(scope="module")
def long92():
    return Case(synth.WORKLOADS["long"])


def _heads_f64(c, names, heads):
    return {n: oracle.bf16_bits_to_f64(c.cpu[n][list(heads)]) for n in names}


def _slice_mask(om, heads):
    return {k: np.ascontiguousarray(v[list(heads)]) for k, v in om.items()}


def _sampled_forward(c, om, gm, heads, blocks_per_head, seed):
    w = c.w
    o, lse = nabla.attn_fwd(c.shape, c.params(), c.gpu["q"], c.gpu["k"], c.gpu["v"], gm)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed)
    x = _heads_f64(c, ("q", "k", "v"), heads)
    sm = _slice_mask(om, heads)
    sel = [(hh, int(i)) for hh in range(len(heads))
           for i in rng.choice(w.nb, blocks_per_head, replace=False)]
    oo, ol = oracle.attn_fwd(x["q"], x["k"], x["v"], sm["row_idx"], sm["row_cnt"], w.scale,
                             sel=sel)
    go = o.view(w.BH, w.nb, L, w.D)
    gl = lse.view(w.BH, w.nb, L)
    got = np.stack([bf16_to_f64(go[heads[hh], i]) for hh, i in sel])
    got_l = np.stack([gl[heads[hh], i].cpu().numpy() for hh, i in sel])
    assert_close(got, oo, "O")
    assert np.max(np.abs(got_l - ol)) < 1e-3
    return o, lse


def test_720p_mask_every_row(train720):
    gm = to_np(train720.gpu_mask())
    om = train720.oracle_mask()
    assert check_mask(gm, om) == 0


def test_720p_debug_scores_cut_only(train720):
    """The kernel's own float32 scores (NABLA_DEBUG_SCORES) equal the oracle's
    score routine bit for bit, and the oracle's cut applied to them gives the
    kernel's mask on every row of all 40 heads."""
    c = train720
    prm = c.params(c.p, nabla.DEBUG_SCORES)
    gm = to_np(nabla.build_mask(c.shape, prm, c.gpu["q"], c.gpu["k"]))
    qb, kb = oracle.pool_f32(c.cpu["q"]), oracle.pool_f32(c.cpu["k"])
    assert np.array_equal(gm["scores"], oracle.scores_f32(qb, kb, c.w.scale))
    om = oracle.mask_from_scores(gm["scores"], c.w.grid_blocks, c.p, c.w.window)
    assert check_mask(gm, om) == 0


def test_720p_forward_sampled(train720):
    om = train720.oracle_mask()
    gm = train720.gpu_mask()
    _sampled_forward(train720, om, gm, heads=(0, 17, 39), blocks_per_head=32, seed=1)


def _key_pairs(w, col_idx, col_cnt, rng, pairs=4):
    """Key blocks for the sampled dK/dV check of one head: `pairs` temporal
    pairs (the same patch in frames 2u and 2u + 1, the unit the dK/dV kernel
    walks together), spatial neighbours of each other so that their column
    lists overlap, plus the pair among a seeded candidate set whose two column
    lists differ the most (the union the kernel walks is then not one list)."""
    T, Hp, Wp = w.grid_blocks
    hw = Hp * Wp

    def pair(u, ph, pw):
        j = (2 * u * Hp + ph) * Wp + pw
        return j, j + hw

    def diff(j0, j1):
        a = set(col_idx[j0, :col_cnt[j0]].tolist())
        b = set(col_idx[j1, :col_cnt[j1]].tolist())
        return len(a ^ b)

    u, ph, pw = int(rng.integers(T // 2)), int(rng.integers(Hp - 1)), int(rng.integers(Wp - 1))
    out = list(pair(u, ph, pw)) + list(pair(u, ph, pw + 1)) + list(pair(u, ph + 1, pw))
    cands = [pair(int(rng.integers(T // 2)), int(rng.integers(Hp)), int(rng.integers(Wp)))
             for _ in range(24)]
    out += list(max(cands, key=lambda jj: diff(*jj)))
    assert diff(out[-2], out[-1]) > 0
    return out[:2 * pairs]


def test_720p_backward_sampled(train720):
    c, w = train720, train720.w
    om = c.oracle_mask()
    gm = c.gpu_mask()
    o, lse = nabla.attn_fwd(c.shape, c.params(), c.gpu["q"], c.gpu["k"], c.gpu["v"], gm)
    dq, dk, dv = nabla.attn_bwd(c.shape, c.params(), c.gpu["q"], c.gpu["k"], c.gpu["v"], o,
                                c.gpu["dout"], lse, gm)
    torch.cuda.synchronize()
    heads = (5, 30)
    x = _heads_f64(c, ("q", "k", "v", "dout"), heads)
    sm = _slice_mask(om, heads)
    rng = np.random.default_rng(2)
    dq_sel = [(hh, int(i)) for hh in range(2) for i in rng.choice(w.nb, 6, replace=False)]
    kv_sel = [(hh, j) for hh in range(2) for j in _key_pairs(w, sm["col_idx"][hh],
                                                             sm["col_cnt"][hh], rng)]
    assert len(kv_sel) == 16
    oq, ok_, ov = oracle.attn_bwd(x["q"], x["k"], x["v"], x["dout"], sm["row_idx"],
                                  sm["row_cnt"], sm["col_idx"], sm["col_cnt"], w.scale,
                                  dq_sel=dq_sel, kv_sel=kv_sel)
    gq = dq.view(w.BH, w.nb, L, w.D)
    gk = dk.view(w.BH, w.nb, L, w.D)
    gv = dv.view(w.BH, w.nb, L, w.D)
    assert_close(np.stack([bf16_to_f64(gq[heads[hh], i]) for hh, i in dq_sel]), oq, "dQ")
    assert_close(np.stack([bf16_to_f64(gk[heads[hh], j]) for hh, j in kv_sel]), ok_, "dK")
    assert_close(np.stack([bf16_to_f64(gv[heads[hh], j]) for hh, j in kv_sel]), ov, "dV")


@pytest.mark.parametrize("p", [0.5, 0.7, 0.9, 1.0])
def test_long_mask_every_row(long92, p):
    gm = to_np(long92.gpu_mask(p))
    om = long92.oracle_mask(p)
    assert check_mask(gm, om) == 0
    if p == 1.0:
        assert np.all(gm["row_cnt"] == long92.w.nb)


@pytest.mark.parametrize("p,heads,blocks", [(0.7, (0, 11), 16), (1.0, (3,), 6)])
def test_long_forward_sampled(long92, p, heads, blocks):
    om = long92.oracle_mask(p)
    gm = long92.gpu_mask(p)
    o, _ = nabla.attn_fwd(long92.shape, long92.params(p), long92.gpu["q"], long92.gpu["k"],
                          long92.gpu["v"], gm)
    torch.cuda.synchronize()
    w = long92.w
    rng = np.random.default_rng(3)
    x = _heads_f64(long92, ("q", "k", "v"), heads)
    sm = _slice_mask(om, heads)
    sel = [(hh, int(i)) for hh in range(len(heads)) for i in rng.choice(w.nb, blocks, replace=False)]
    oo, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], sm["row_idx"], sm["row_cnt"], w.scale, sel=sel)
    go = o.view(w.BH, w.nb, L, w.D)
    assert_close(np.stack([bf16_to_f64(go[heads[hh], i]) for hh, i in sel]), oo, "O")


@pytest.fixture(scope="module")
def max2048():
    # the largest block count the library accepts: T=32, 64x64 latent -> 32 x 8 x 8 = 2048
    # blocks of 64 tokens (131,072 tokens), one head, with a training backward
    return Case(synth.Workload("max2048", 1, 1, 32, 64, 64, 128, (2, 8, 8), 0.7, backward=True))


def test_max_blocks_mask_every_row(max2048):
    assert max2048.w.nb == 2048
    gm = to_np(max2048.gpu_mask())
    om = max2048.oracle_mask()
    assert check_mask(gm, om) == 0


def test_max_blocks_forward_and_backward_sampled(max2048):
    c, w = max2048, max2048.w
    om = c.oracle_mask()
    gm = c.gpu_mask()
    o, lse = _sampled_forward(c, om, gm, heads=(0,), blocks_per_head=12, seed=4)
    dq, dk, dv = nabla.attn_bwd(c.shape, c.params(), c.gpu["q"], c.gpu["k"], c.gpu["v"], o,
                                c.gpu["dout"], lse, gm)
    torch.cuda.synchronize()
    x = _heads_f64(c, ("q", "k", "v", "dout"), (0,))
    rng = np.random.default_rng(5)
    dq_sel = [(0, int(i)) for i in rng.choice(w.nb, 6, replace=False)]
    kv_sel = [(0, 0), (0, w.nb - 1)]  # the first and the last key block
    oq, ok_, ov = oracle.attn_bwd(x["q"], x["k"], x["v"], x["dout"], om["row_idx"], om["row_cnt"],
                                  om["col_idx"], om["col_cnt"], w.scale, dq_sel=dq_sel,
                                  kv_sel=kv_sel)
    gq = dq.view(w.BH, w.nb, L, w.D)
    gk = dk.view(w.BH, w.nb, L, w.D)
    gv = dv.view(w.BH, w.nb, L, w.D)
    assert_close(np.stack([bf16_to_f64(gq[0, i]) for _, i in dq_sel]), oq, "dQ")
    assert_close(np.stack([bf16_to_f64(gk[0, j]) for _, j in kv_sel]), ok_, "dK")
    assert_close(np.stack([bf16_to_f64(gv[0, j]) for _, j in kv_sel]), ov, "dV")

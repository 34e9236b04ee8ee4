"""nabla_build_mask_dr (DynamicRad-style masks, "DynamicRad: Content-Adaptive
Sparse Attention for Long Video Diffusion", section 2.A) on the GPU against
the oracle: bit rows, row lists and column lists bit-exact on every row, for
the static-ratio mode (several decay / floor settings, grids with patch grids
narrower and wider than a warp, one frame) and the logit-threshold mode (with
its scores checked bit for bit through NABLA_DEBUG_SCORES); then the same
attention forward and backward consuming such a mask, against the float64
oracle within max-abs 2e-2 / mean-abs 2e-3."""
import numpy as np
import pytest
import torch

import oracle
from adaptive_block_sparse_fractal_b200 import nabla, synth

from gpu_util import Case, assert_close, bf16_to_f64, check_mask, f64, list_equal, to_np

pytestmark = pytest.mark.gpu

SHAPES = [
    synth.WORKLOADS["tiny"],
    synth.Workload("odd130", 2, 2, 5, 16, 104, 128, (2, 4, 4), 0.7),   # Wp = 13, ragged tile
    synth.Workload("w40", 1, 1, 3, 16, 320, 64, (1, 4, 4), 0.7),       # Wp = 40 > a warp
    synth.Workload("one_frame", 1, 2, 1, 32, 32, 128, (1, 4, 4), 0.7),  # T = 1
    synth.WORKLOADS["small"],
]


def _exact(gm, om):
    """Every row bit-exact (no decision here is within rounding of a cut)."""
    assert np.array_equal(gm["bits"], om["bits"])
    assert list_equal(gm["row_idx"], gm["row_cnt"], om["row_idx"], om["row_cnt"])
    assert list_equal(gm["col_idx"], gm["col_cnt"], om["col_idx"], om["col_cnt"])


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
@pytest.mark.parametrize("gamma,lam,flags", [(0.6, 0.1, 0), (0.85, 0.0, nabla.NO_STA),
                                             (1e-9, 0.0, 0), (1.0, 0.0, nabla.NO_STA)])
def test_static_ratio_every_row(w, gamma, lam, flags):
    shape = nabla.shape_of(w.B, w.heads, w.T, w.H, w.W, w.D, w.P)
    prm = nabla.dr_params_of(nabla.DR_STATIC_RATIO, gamma, lam, window=w.window, D=w.D,
                             flags=flags | nabla.EMIT_COLS)
    gm = to_np(nabla.build_mask_dr(shape, prm, device=torch.device("cuda")))
    om = oracle.dr_static(w.BH, w.grid_blocks, gamma, lam, w.window, flags)
    _exact(gm, om)


def _threshold(c, tau, flags=0):
    w = c.w
    prm = nabla.dr_params_of(nabla.DR_THRESHOLD, tau=tau, window=w.window, D=w.D,
                             flags=flags | nabla.EMIT_COLS | nabla.DEBUG_SCORES)
    gm = to_np(nabla.build_mask_dr(c.shape, prm, c.gpu["q"], c.gpu["k"]))
    qb, kb = oracle.pool_f32(c.cpu["q"]), oracle.pool_f32(c.cpu["k"])
    assert np.array_equal(gm["scores"], oracle.scores_f32(qb, kb, w.scale))
    om = oracle.dr_threshold(qb, kb, w.grid_blocks, tau, w.scale, w.window, flags)
    _exact(gm, om)
    return gm


@pytest.mark.parametrize("w", [s for s in SHAPES if s.name != "w40"], ids=lambda w: w.name)
@pytest.mark.parametrize("tau,flags", [(0.0, nabla.NO_STA), (0.4, 0), (1.5, nabla.NO_STA),
                                       (float("inf"), 0)])
def test_threshold_every_row(w, tau, flags):
    gm = _threshold(Case(w), tau, flags)
    if tau == float("inf"):
        assert np.all(gm["row_cnt"] == w.nb)


@pytest.fixture(scope="module")
def train720():
    return Case(synth.WORKLOADS["train"], backward=False)


def test_720p_both_modes_every_row(train720):
    c, w = train720, train720.w
    _threshold(c, 1.0)
    prm = nabla.dr_params_of(nabla.DR_STATIC_RATIO, 0.7, 0.05, window=w.window, D=w.D,
                             flags=nabla.EMIT_COLS)
    gm = to_np(nabla.build_mask_dr(c.shape, prm, device=torch.device("cuda")))
    _exact(gm, oracle.dr_static(w.BH, w.grid_blocks, 0.7, 0.05, w.window))


@pytest.mark.parametrize("mode", [nabla.DR_STATIC_RATIO, nabla.DR_THRESHOLD])
def test_attention_over_a_dynamicrad_mask(mode):
    # the ragged 130-block shape, D = 128 (tcgen05 kernels), full forward and backward
    w = synth.Workload("odd130", 2, 2, 5, 16, 104, 128, (2, 4, 4), 0.7, backward=True)
    c = Case(w)
    prm = nabla.dr_params_of(mode, 0.6, 0.1, tau=0.8, window=w.window, D=w.D,
                             flags=nabla.EMIT_COLS)
    if mode == nabla.DR_THRESHOLD:
        m = nabla.build_mask_dr(c.shape, prm, c.gpu["q"], c.gpu["k"])
        om = oracle.dr_threshold(oracle.pool_f32(c.cpu["q"]), oracle.pool_f32(c.cpu["k"]),
                                 w.grid_blocks, 0.8, w.scale, w.window)
    else:
        m = nabla.build_mask_dr(c.shape, prm, device=torch.device("cuda"))
        om = oracle.dr_static(w.BH, w.grid_blocks, 0.6, 0.1, w.window)
    kept = float(om["row_cnt"].sum()) / (w.BH * w.nb * w.nb)
    assert 0.05 < kept < 0.95  # a sparse mask
    ap = c.params()
    o, lse = nabla.attn_fwd(c.shape, ap, c.gpu["q"], c.gpu["k"], c.gpu["v"], m)
    dq, dk, dv = nabla.attn_bwd(c.shape, ap, c.gpu["q"], c.gpu["k"], c.gpu["v"], o, c.gpu["dout"],
                                lse, m)
    torch.cuda.synchronize()
    x = {n: f64(c.cpu[n]) for n in ("q", "k", "v", "dout")}
    oo, ol = oracle.attn_fwd(x["q"], x["k"], x["v"], om["row_idx"], om["row_cnt"], w.scale)
    gq, gk, gv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["dout"], om["row_idx"], om["row_cnt"],
                                 om["col_idx"], om["col_cnt"], w.scale)
    assert_close(bf16_to_f64(o).reshape(oo.shape), oo, "O")
    assert np.abs(lse.cpu().numpy().reshape(ol.shape) - ol).max() < 1e-3
    assert_close(bf16_to_f64(dq).reshape(gq.shape), gq, "dQ")
    assert_close(bf16_to_f64(dk).reshape(gk.shape), gk, "dK")
    assert_close(bf16_to_f64(dv).reshape(gv.shape), gv, "dV")

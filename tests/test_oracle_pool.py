"""Pins of the oracle's block mean-pooling (NABLA page, 手法: NABLA, bullet
"ダウンサンプリング": Q and K are reshaped and mean-pooled into blocks).  A
block is one P x P patch of one frame, i.e. 64 consecutive flattened tokens."""
import numpy as np
import torch

from adaptive_block_sparse_fractal_b200 import synth


def _bf16_bits(a):
    return synth.bits(torch.as_tensor(a, dtype=torch.float32).to(torch.bfloat16))


def test_constant_blocks_pool_to_the_constant(oracle_mod):
    BH, nb, D = 2, 5, 16
    rng = np.random.default_rng(0)
    c = rng.standard_normal((BH, nb, 1, D)).astype(np.float32)
    c = (torch.tensor(c).to(torch.bfloat16).float().numpy())  # representable
    x = np.broadcast_to(c, (BH, nb, 64, D)).reshape(BH, nb * 64, D)
    xb = _bf16_bits(x)
    assert np.array_equal(oracle_mod.pool_f32(xb), c[:, :, 0, :])
    assert np.array_equal(oracle_mod.pool_f64(xb), c[:, :, 0, :].astype(np.float64))


def test_ramp_pools_to_its_midpoint(oracle_mod):
    BH, nb, D = 1, 3, 4
    r = np.arange(64, dtype=np.float32)
    x = np.tile(r[None, :, None], (nb, 1, D)).reshape(1, nb * 64, D)
    x = x + 100.0 * np.repeat(np.arange(nb), 64)[None, :, None]
    xb = _bf16_bits(x)
    want = 31.5 + 100.0 * np.arange(nb)[None, :, None] * np.ones((1, 1, D))
    assert np.array_equal(oracle_mod.pool_f64(xb), want)
    assert np.array_equal(oracle_mod.pool_f32(xb), want.astype(np.float32))


def test_pool_is_the_patch_mean_in_grid_layout(oracle_mod):
    # Pooling the flattened sequence equals averaging each P x P patch of each
    # frame directly on the [T, H, W, D] grid (numpy reshape + mean).
    T, H, W, P, D = 2, 16, 24, 8, 8
    x = synth.cell_correlated(1, 1, T, H, W, D, (2, 4, 4), seed=3)
    g = x[0, 0].float().numpy().astype(np.float64)
    want = g.reshape(T, H // P, P, W // P, P, D).mean(axis=(2, 4)).reshape(-1, D)
    flat = oracle_mod.flatten_tokens(synth.bits(x).reshape(1, T * H * W, D), T, H, W, P)
    got = oracle_mod.pool_f64(flat)[0]
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_f32_decision_pool_tracks_f64(oracle_mod):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 64 * 7, 32)).astype(np.float32) * 3
    xb = _bf16_bits(x)
    a, b = oracle_mod.pool_f32(xb), oracle_mod.pool_f64(xb)
    assert np.max(np.abs(a - b)) < 1e-5
    # block means are invariant to the order of tokens inside a block (float64
    # sums of bf16 values are exact here)
    perm = rng.permutation(64)
    xp = xb.reshape(3, 7, 64, 32)[:, :, perm].reshape(3, 7 * 64, 32)
    assert np.array_equal(oracle_mod.pool_f64(xp), b)

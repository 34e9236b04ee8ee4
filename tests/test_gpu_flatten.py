"""nabla_flatten on the GPU vs the oracle's permutation: bit-exact, both
directions, several grids (ragged patch counts), element sizes and outer
dims, including [B, T, H, W, C] activations."""
import numpy as np
import pytest
import torch

import oracle
from adaptive_block_sparse_fractal_b200 import nabla

pytestmark = pytest.mark.gpu

GRIDS = [(4, 16, 16, 8), (3, 16, 24, 8), (1, 8, 8, 8), (2, 48, 80, 8), (5, 8, 40, 8),
         (2, 12, 18, 6), (3, 4, 4, 2)]


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("inner", [16, 128, 256, 48])
def test_flatten_bit_exact(grid, inner):
    T, H, W, P = grid
    rng = np.random.default_rng(hash((grid, inner)) % 2**32)
    outer = 3
    x = rng.integers(0, 256, size=(outer, T * H * W, inner), dtype=np.uint8)
    want = oracle.flatten(x, T, H, W, P)
    xg = torch.from_numpy(x).cuda()
    got = nabla.flatten(xg, T, H, W, P).cpu().numpy()
    assert np.array_equal(got, want)
    back = nabla.flatten(torch.from_numpy(want).cuda(), T, H, W, P, inverse=True).cpu().numpy()
    assert np.array_equal(back, x)


def test_flatten_activations_layout():
    # [B, T, H, W, C] bf16 activations: outer = B, inner = C
    B, T, H, W, C = 2, 3, 16, 24, 320
    x = torch.randn(B, T, H, W, C).to(torch.bfloat16)
    f = nabla.flatten(x.cuda(), T, H, W, 8)
    want = oracle.flatten(x.view(torch.int16).numpy().reshape(B, T * H * W, C).view(np.uint8),
                          T, H, W, 8)
    assert np.array_equal(f.cpu().view(torch.int16).numpy().reshape(B, -1, C).view(np.uint8),
                          want)


def test_flatten_twice_is_deterministic_and_empty_is_noop():
    x = torch.randint(0, 255, (2, 4 * 16 * 16, 256), dtype=torch.uint8, device="cuda")
    a = nabla.flatten(x, 4, 16, 16)
    b = nabla.flatten(x, 4, 16, 16)
    assert torch.equal(a, b)
    e = torch.empty((0, 64, 16), dtype=torch.uint8, device="cuda")
    assert nabla.flatten(e, 1, 8, 8).numel() == 0

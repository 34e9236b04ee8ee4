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


def test_pooled_means_bit_exact(small):
    w = small.w
    ws = nabla.workspace(small.shape, nabla.OP_BUILD_MASK, "cuda")
    nabla.build_mask(small.shape, small.params(), small.gpu["q"], small.gpu["k"], ws=ws)
    torch.cuda.synchronize()
    n = w.BH * w.nb * w.D
    raw = ws.cpu().numpy()
    qbar = raw[256:256 + 4 * n].view(np.float32).reshape(w.BH, w.nb, w.D)
    off = 256 + ((4 * n + 255) // 256) * 256
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

"""Seeded synthetic inputs shaped like video-diffusion attention activations.

This module holds no arithmetic of the attention method: it only draws
numbers.  Both the CUDA path and the CPU oracle consume what it returns.

Q, K and V are "cell-correlated": the latent grid T x H x W is cut into cells
of ct x cy x cx tokens; every token of a cell shares one N(0, 1)^D vector, and
each token adds its own 0.5 * N(0, 1)^D noise.  Values are cast to bf16 with
round-to-nearest-even, in grid order [B, h, T, H, W, D].  dO is N(0, 1) bf16,
drawn directly in the flattened token order [B, h, N, D].  Seeds: Q, K, V use
seed0 + 1, 2, 3 and dO uses seed0 + 4.
"""
from dataclasses import dataclass, field
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    T: int
    H: int
    W: int
    D: int
    cell: tuple
    p: float
    window: tuple = (3, 3, 3)
    P: int = 8
    noise: float = 0.5
    backward: bool = False
    p_sweep: tuple = field(default_factory=tuple)

    @property
    def N(self):
        return self.T * self.H * self.W

    @property
    def BH(self):
        return self.B * self.heads

    @property
    def nb(self):
        return self.N // (self.P * self.P)

    @property
    def grid_blocks(self):
        return (self.T, self.H // self.P, self.W // self.P)

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.D)


# The five workloads: a tiny check case, a small one, a 720p-like video latent
# (76,800 tokens), the same shape trained (forward + backward), and a long clip
# (92,160 tokens) swept over p.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 4, 16, 16, 64, (2, 4, 4), 0.9),
    "small": Workload("small", 1, 24, 8, 32, 32, 128, (2, 4, 4), 0.8),
    "720p": Workload("720p", 1, 40, 20, 48, 80, 128, (2, 8, 8), 0.7),
    "train": Workload("train", 1, 40, 20, 48, 80, 128, (2, 8, 8), 0.7, backward=True),
    "long": Workload("long", 1, 12, 60, 32, 48, 128, (2, 4, 4), 0.7,
                     p_sweep=(0.5, 0.7, 0.9, 1.0)),
}


def cell_correlated(B, heads, T, H, W, D, cell, seed, noise=0.5, dtype=torch.bfloat16):
    """[B, heads, T, H, W, D] bf16 on the CPU, deterministic in `seed`."""
    g = torch.Generator().manual_seed(int(seed))
    ct, cy, cx = cell
    nct, ncy, ncx = -(-T // ct), -(-H // cy), -(-W // cx)
    c = torch.randn(B, heads, nct, ncy, ncx, D, generator=g, dtype=torch.float32)
    c = (c.repeat_interleave(ct, 2).repeat_interleave(cy, 3).repeat_interleave(cx, 4)
         [:, :, :T, :H, :W])
    x = torch.randn(B, heads, T, H, W, D, generator=g, dtype=torch.float32)
    x.mul_(noise).add_(c)
    return x.to(dtype)


def normal_flat(B, heads, N, D, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(B, heads, N, D, generator=g, dtype=torch.float32).to(dtype)


def make_inputs(w: Workload, seed0: int = 0, heads=None, with_dout=None):
    """Returns dict q, k, v in grid order [B, h, T, H, W, D] (bf16, CPU) and,
    when the workload trains (or with_dout), dout in flattened order
    [B, h, N, D].  `heads` restricts generation to a subset of head indices
    (the draws for other heads are still consumed so values do not depend on
    the subset)."""
    out = {}
    for name, off in (("q", 1), ("k", 2), ("v", 3)):
        out[name] = cell_correlated(w.B, w.heads, w.T, w.H, w.W, w.D, w.cell, seed0 + off,
                                    w.noise)
    if with_dout or (with_dout is None and w.backward):
        out["dout"] = normal_flat(w.B, w.heads, w.N, w.D, seed0 + 4)
    if heads is not None:
        out = {k: v[:, list(heads)].contiguous() for k, v in out.items()}
    return out


def bits(t: torch.Tensor):
    """Raw uint16 bits of a bf16 tensor as a numpy array (same shape)."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def make_inputs_device(w: Workload, seed0: int = 0, device="cuda", with_dout=None,
                       head_range=None):
    """Same recipe as make_inputs, drawn with a generator on `device` (fast for
    the benchmark's full-size workloads; the values differ from the CPU
    stream).  Every (batch, head) slice is drawn from its own seed, so any
    subset of heads is the same as the corresponding slice of the whole
    problem: `head_range` = (h0, h1) draws heads h0 .. h1 - 1 of every batch
    element only (a partition of the heads over devices).  Q, K, V in grid
    order [B*nh, T*H*W, D], dout in flattened order [B*nh, N, D], nh = h1 - h0."""
    h0, h1 = (0, w.heads) if head_range is None else head_range
    assert 0 <= h0 < h1 <= w.heads
    g = torch.Generator(device=device)
    ct, cy, cx = w.cell
    nct, ncy, ncx = -(-w.T // ct), -(-w.H // cy), -(-w.W // cx)
    sel = [b * w.heads + h for b in range(w.B) for h in range(h0, h1)]
    out = {}
    for name, off in (("q", 1), ("k", 2), ("v", 3)):
        x = torch.empty(len(sel), w.N, w.D, dtype=torch.bfloat16, device=device)
        for n, bh in enumerate(sel):
            g.manual_seed(int((seed0 + off) * 100003 + bh))
            c = torch.randn(nct, ncy, ncx, w.D, generator=g, device=device)
            c = (c.repeat_interleave(ct, 0).repeat_interleave(cy, 1).repeat_interleave(cx, 2)
                 [:w.T, :w.H, :w.W])
            t = torch.randn(w.T, w.H, w.W, w.D, generator=g, device=device)
            t.mul_(w.noise).add_(c)
            x[n] = t.to(torch.bfloat16).reshape(w.N, w.D)
            del c, t
        out[name] = x
    if with_dout or (with_dout is None and w.backward):
        x = torch.empty(len(sel), w.N, w.D, dtype=torch.bfloat16, device=device)
        for n, bh in enumerate(sel):
            g.manual_seed(int((seed0 + 4) * 100003 + bh))
            x[n] = torch.randn(w.N, w.D, generator=g, device=device).to(torch.bfloat16)
        out["dout"] = x
    return out

"""Shared helpers of the GPU parity tests: identical seeded inputs for the
CUDA path (flattened on the GPU by nabla_flatten) and the oracle (flattened on
the CPU by its own loops), and the comparison rules.

Tolerance for bf16 outputs and gradients (fp32 accumulation) against the
float64 oracle: max-abs <= 2e-2 and mean-abs <= 2e-3.  Masks and
permutations: bit-exact."""
import numpy as np
import torch

import oracle
from adaptive_block_sparse_fractal_b200 import nabla, synth

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
FRAGILE_UNITS = 64.0  # a cut decided within 64 units of 2^-40 mass


class Case:
    """A workload with inputs on both sides."""

    def __init__(self, w, seed0=0, p=None, flags=0, backward=None, device="cuda", mutate=None):
        self.w = w
        self.p = w.p if p is None else p
        self.flags = flags
        self.backward = w.backward if backward is None else backward
        inp = synth.make_inputs(w, seed0, with_dout=self.backward)
        if mutate is not None:  # a test's deliberate change to the inputs, applied to both sides
            mutate(inp)
        self.shape = nabla.shape_of(w.B, w.heads, w.T, w.H, w.W, w.D, w.P)
        self.cpu = {}
        self.gpu = {}
        for name in ("q", "k", "v"):
            grid_bits = synth.bits(inp[name]).reshape(w.BH, w.N, w.D)
            self.cpu[name] = oracle.flatten_tokens(grid_bits, w.T, w.H, w.W, w.P)
            g = inp[name].reshape(w.BH, w.N, w.D).to(device)
            self.gpu[name] = nabla.flatten(g, w.T, w.H, w.W, w.P)
            del g
        if self.backward:
            self.cpu["dout"] = synth.bits(inp["dout"]).reshape(w.BH, w.N, w.D)
            self.gpu["dout"] = inp["dout"].reshape(w.BH, w.N, w.D).to(device)
        torch.cuda.synchronize()

    def params(self, p=None, flags=None):
        f = (self.flags if flags is None else flags) | nabla.EMIT_COLS
        return nabla.params_of(self.p if p is None else p, self.w.window, D=self.w.D, flags=f)

    def oracle_mask(self, p=None, flags=None):
        return oracle.build_mask(self.cpu["q"], self.cpu["k"], self.w.grid_blocks,
                                 self.p if p is None else p, self.w.scale, self.w.window,
                                 self.flags if flags is None else flags)

    def gpu_mask(self, p=None, flags=None):
        return nabla.build_mask(self.shape, self.params(p, flags), self.gpu["q"], self.gpu["k"])


def to_np(m):
    out = {}
    for k, t in m.items():
        a = t.cpu().numpy()
        if k in ("row_idx", "col_idx"):
            a = a.view(np.uint16)
        if k == "bits":
            a = a.view(np.uint32)
        out[k] = a
    return out


def list_equal(idx_a, cnt_a, idx_b, cnt_b, rows=None):
    """Compare fixed-stride lists on the written prefix only."""
    nb = idx_a.shape[-1]
    if rows is None:
        rows = np.ones(cnt_a.shape, dtype=bool)
    if not np.array_equal(cnt_a[rows], cnt_b[rows]):
        return False
    valid = (np.arange(nb)[None, None, :] < cnt_a[..., None]) & rows[..., None]
    return np.array_equal(np.where(valid, idx_a, 0), np.where(valid, idx_b, 0))


def check_mask(gm, om):
    """GPU mask (numpy) vs oracle mask: bit-exact on every row whose cut is
    not within FRAGILE_UNITS of the threshold; the GPU lists must match its
    own bits everywhere.  Returns the number of fragile rows."""
    fragile = om["margin"] <= FRAGILE_UNITS
    solid = ~fragile
    assert np.array_equal(gm["bits"][solid], om["bits"][solid]), "bit rows differ"
    assert list_equal(gm["row_idx"], gm["row_cnt"], om["row_idx"], om["row_cnt"], solid)
    # structural: lists are the bits, columns are their transpose
    BH, nb = gm["row_cnt"].shape
    dense = np.unpackbits(gm["bits"].view(np.uint8), axis=-1, bitorder="little")[..., :nb]
    dense = dense.astype(bool)
    assert np.array_equal(gm["row_cnt"], dense.sum(-1))
    if "col_cnt" in gm:
        assert np.array_equal(gm["col_cnt"], dense.sum(-2))
        if not fragile.any():
            assert list_equal(gm["col_idx"], gm["col_cnt"], om["col_idx"], om["col_cnt"])
    return int(fragile.sum())


def err_stats(got, want):
    d = np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))
    return float(d.max()), float(d.mean())


def assert_close(got, want, what):
    mx, mean = err_stats(got, want)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, "%s: max-abs %.3g mean-abs %.3g" % (what, mx, mean)
    return mx, mean


def f64(bits):
    return oracle.bf16_bits_to_f64(bits)


def bf16_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)

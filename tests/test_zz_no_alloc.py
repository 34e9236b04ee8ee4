"""nabla_build_mask_static: the mask build for callers that cannot allocate.

Some callers get only their input and output buffers (a plugin interface
with no workspace argument, or a process whose device memory another
allocator reserved up front) and cannot call cudaMalloc for the pooled-mean
scratch that nabla_build_mask takes as a workspace.  This entry point keeps
that scratch in an array compiled into the library instead.  The test calls
it through the C ABI twice in a row, on two different problems, and checks
every output against the workspace entry point bit for bit (masks are integer
results: the tolerance the other mask tests use is exact equality).  It also
checks that a problem larger than the built-in scratch is refused.

This file is collected last on purpose, and passes both alone in a fresh
process and after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

from adaptive_block_sparse_fractal_b200 import nabla, synth

pytestmark = pytest.mark.gpu


def _problem(w, seed, flags=nabla.EMIT_COLS):
    dev = torch.device("cuda")
    g = synth.make_inputs_device(w, seed, dev, with_dout=False)
    q = nabla.flatten(g["q"], w.T, w.H, w.W, w.P)
    k = nabla.flatten(g["k"], w.T, w.H, w.W, w.P)
    shape = nabla.shape_of(w.B, w.heads, w.T, w.H, w.W, w.D, w.P)
    prm = nabla.params_of(w.p, w.window, D=w.D, flags=flags)
    return shape, prm, q, k


def _static_call(shape, prm, q, k, mask):
    ms = nabla._mask_struct(mask)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return nabla.lib().nabla_build_mask_static(ctypes.byref(shape), ctypes.byref(prm),
                                              ctypes.c_void_p(q.data_ptr()),
                                              ctypes.c_void_p(k.data_ptr()), ctypes.byref(ms),
                                              stream)


def _same(a, b):
    nb = a["row_cnt"].shape[-1]
    cols = "col_cnt" in b
    assert cols == ("col_cnt" in a)
    for key in ("bits", "row_cnt") + (("col_cnt",) if cols else ()):
        assert torch.equal(a[key], b[key]), key
    for idx, cnt in (("row_idx", "row_cnt"),) + ((("col_idx", "col_cnt"),) if cols else ()):
        valid = torch.arange(nb, device=a[idx].device)[None, None, :] < a[cnt][..., None]
        assert torch.equal(torch.where(valid, a[idx], 0), torch.where(valid, b[idx], 0)), idx


def test_static_scratch_matches_workspace_entry_point_twice():
    small = synth.WORKLOADS["small"]
    odd = synth.Workload("odd130", 2, 2, 5, 16, 104, 128, (2, 4, 4), 0.7)
    tiny = synth.WORKLOADS["tiny"]  # D = 64, no column lists
    # calls in a row, different shapes
    for w, seed, flags in ((small, 0, nabla.EMIT_COLS), (odd, 5, nabla.EMIT_COLS), (tiny, 2, 0)):
        shape, prm, q, k = _problem(w, seed, flags)
        want = nabla.build_mask(shape, prm, q, k)
        got = nabla.alloc_mask(shape, q.device, cols=bool(flags & nabla.EMIT_COLS))
        for key in got:
            got[key].fill_(-1)  # stale contents must not leak into the result
        assert _static_call(shape, prm, q, k, got) == nabla.OK
        torch.cuda.synchronize()
        _same(got, want)
        assert int(want["row_cnt"].sum()) > w.BH * w.nb  # a real, non-trivial mask


def test_static_scratch_refuses_oversize_problem():
    w = synth.WORKLOADS["720p"]  # pooled means need ~47 MiB > 32 MiB
    shape = nabla.shape_of(w.B, w.heads, w.T, w.H, w.W, w.D, w.P)
    prm = nabla.params_of(w.p, w.window, D=w.D, flags=0)
    tiny = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    m = {k: torch.empty(4, dtype=torch.int32, device="cuda") for k in ("bits", "row_idx", "row_cnt")}
    assert _static_call(shape, prm, tiny, tiny, m) == nabla.ERR_WORKSPACE

"""The C-ABI library without a GPU: it loads, exports every function that
include/nabla.h declares, sizes buffers as documented, and rejects invalid
arguments on the host before enqueuing anything (fault injection on the
host: bad shapes, parameters, NULL and misaligned pointers, short
workspaces)."""
import ctypes
import os
import re

import pytest

from adaptive_block_sparse_fractal_b200 import build, nabla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return nabla.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "nabla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(nabla_[a-z_]+)\s*\(", src))


def test_exports_every_declared_symbol(L):
    declared = _declared()
    assert declared == set(nabla.SYMBOLS)
    for name in declared:
        assert hasattr(L, name), name


def test_strerror(L):
    for st in (0, -1, -2, -3, -4, -5, -6, -7):
        assert nabla.strerror(st) and nabla.strerror(st) != "unknown status"
    assert nabla.strerror(-99) == "unknown status"


def _shape(**kw):
    d = dict(B=1, heads=40, T=20, H=48, W=80, D=128, P=8)
    d.update(kw)
    return nabla.Shape(*(d[k] for k in ("B", "heads", "T", "H", "W", "D", "P")))


def test_sizes(L):
    s = _shape()
    BH, nb, N, D = 40, 1200, 76800, 128
    assert nabla.mask_bytes(s, nabla.MASK_BITS) == BH * nb * ((nb + 31) // 32) * 4
    assert nabla.mask_bytes(s, nabla.MASK_ROW_IDX) == BH * nb * nb * 2
    assert nabla.mask_bytes(s, nabla.MASK_COL_CNT) == BH * nb * 4
    # status word, task counters of the persistent front end, pooled Q and K
    ctr = (4 * (1 + BH) + 255) // 256 * 256
    assert nabla.workspace_size(s, nabla.OP_BUILD_MASK) == 256 + ctr + 2 * BH * nb * D * 4
    assert nabla.workspace_size(s, nabla.OP_ATTN_BWD) == 256 + 2 * BH * N * 4
    assert nabla.workspace_size(s, nabla.OP_ATTN_FWD) >= 256
    # invalid shapes size to 0
    for bad in (_shape(P=4), _shape(D=96), _shape(H=50), _shape(T=0), _shape(T=200)):
        assert nabla.workspace_size(bad, nabla.OP_BUILD_MASK) == 0
        assert nabla.mask_bytes(bad, nabla.MASK_BITS) == 0


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails validation
FAKE_ODD = ctypes.c_void_p(0x10008)


def _mask():
    return nabla.MaskStruct(FAKE, FAKE, FAKE, FAKE, FAKE)


def _build(L, shape, params, q=FAKE, k=FAKE, mask=None, ws=FAKE, ws_bytes=1 << 40):
    m = _mask() if mask is None else mask
    return L.nabla_build_mask(ctypes.byref(shape), ctypes.byref(params), q, k, ctypes.byref(m),
                              ws, ws_bytes, None)


def test_build_mask_rejects_on_host(L):
    good = nabla.params_of(0.7, (3, 3, 3), D=128)
    assert _build(L, _shape(H=44), good) == nabla.ERR_SHAPE
    assert _build(L, _shape(D=32), good) == nabla.ERR_SHAPE
    for p in (-0.1, 1.5, float("nan")):
        assert _build(L, _shape(), nabla.params_of(p, (3, 3, 3), D=128)) == nabla.ERR_PARAM
    assert _build(L, _shape(), nabla.params_of(0.5, (2, 3, 3), D=128)) == nabla.ERR_PARAM
    assert _build(L, _shape(), nabla.params_of(0.5, (3, 3, 0), D=128)) == nabla.ERR_PARAM
    assert _build(L, _shape(), nabla.params_of(0.5, (3, 3, 3), scale=0.0)) == nabla.ERR_PARAM
    both = nabla.params_of(0.5, (3, 3, 3), D=128, flags=nabla.NO_STA | nabla.FULL_STA)
    assert _build(L, _shape(), both) == nabla.ERR_PARAM
    # even windows are fine when the STA term is off
    nosta = nabla.params_of(0.5, (2, 2, 2), D=128, flags=nabla.NO_STA)
    assert _build(L, _shape(), nosta, q=None) == nabla.ERR_NULL
    assert _build(L, _shape(), good, k=None) == nabla.ERR_NULL
    cols = nabla.params_of(0.5, (3, 3, 3), D=128, flags=nabla.EMIT_COLS)
    assert _build(L, _shape(), cols, mask=nabla.MaskStruct(FAKE, FAKE, FAKE, None, None)) == \
        nabla.ERR_NULL
    assert _build(L, _shape(), good, q=FAKE_ODD) == nabla.ERR_ALIGN
    assert _build(L, _shape(), good, ws=None) == nabla.ERR_WORKSPACE
    assert _build(L, _shape(), good, ws_bytes=1024) == nabla.ERR_WORKSPACE
    assert _build(L, _shape(), good, ws=FAKE_ODD) == nabla.ERR_ALIGN
    assert L.nabla_build_mask(None, ctypes.byref(good), FAKE, FAKE, ctypes.byref(_mask()), FAKE,
                              1 << 40, None) == nabla.ERR_NULL


def test_build_mask_grid_rejects_on_host(L):
    s, good = _shape(), nabla.params_of(0.7, (3, 3, 3), D=128)
    bytes_ = 2 * s.B * s.heads * s.T * s.H * s.W * s.D
    a, b = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000 + bytes_)
    c, d = ctypes.c_void_p(0x10000 + 2 * bytes_), ctypes.c_void_p(0x10000 + 3 * bytes_)

    def g(qg, kg, q, k, mask=None, params=good, ws_bytes=1 << 40):
        m = _mask() if mask is None else mask
        return L.nabla_build_mask_grid(ctypes.byref(s), ctypes.byref(params), qg, kg, q, k,
                                       ctypes.byref(m), FAKE, ws_bytes, None)
    assert g(None, b, c, d) == nabla.ERR_NULL
    assert g(a, b, c, None) == nabla.ERR_NULL
    assert g(a, b, FAKE_ODD, d) == nabla.ERR_ALIGN
    assert g(a, b, c, c) == nabla.ERR_PARAM                                  # q overlaps k
    assert g(a, b, a, d) == nabla.ERR_PARAM                                  # in place
    assert g(a, b, ctypes.c_void_p(0x10000 + bytes_ // 2), d) == nabla.ERR_PARAM  # partial overlap
    assert g(a, b, c, d, ws_bytes=1024) == nabla.ERR_WORKSPACE
    assert g(a, b, c, d, params=nabla.params_of(1.5, (3, 3, 3), D=128)) == nabla.ERR_PARAM


def test_debug_scores_needs_its_buffer(L):
    s = _shape()
    assert nabla.mask_bytes(s, nabla.MASK_SCORES) == 40 * 1200 * 1200 * 4
    dbg = nabla.params_of(0.7, (3, 3, 3), D=128, flags=nabla.DEBUG_SCORES)
    assert _build(L, s, dbg) == nabla.ERR_NULL  # mask.scores is NULL
    m = nabla.MaskStruct(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert _build(L, s, dbg, mask=m, ws_bytes=1024) == nabla.ERR_WORKSPACE  # got past the NULL check


def _dr(L, params, shape=None, q=FAKE, k=FAKE, mask=None, ws=FAKE, ws_bytes=1 << 40):
    m = _mask() if mask is None else mask
    s = _shape() if shape is None else shape
    return L.nabla_build_mask_dr(ctypes.byref(s), ctypes.byref(params), q, k, ctypes.byref(m), ws,
                                 ws_bytes, None)


def test_dynamicrad_masks_reject_on_host(L):
    ratio = lambda **kw: nabla.dr_params_of(nabla.DR_STATIC_RATIO, D=128, **kw)
    thr = lambda **kw: nabla.dr_params_of(nabla.DR_THRESHOLD, D=128, **kw)
    for bad in (ratio(gamma=0.0), ratio(gamma=1.5), ratio(gamma=0.5, lam=-0.1),
                ratio(gamma=0.5, lam=1.1), thr(tau=-1.0), thr(tau=float("nan")),
                ratio(gamma=0.5, window=(2, 3, 3)),
                ratio(gamma=0.5, flags=nabla.DEBUG_SCORES),  # the static mode has no scores
                thr(tau=1.0, flags=nabla.DEBUG_TIMEOUT)):
        assert _dr(L, bad) == nabla.ERR_PARAM
    bad_mode = thr(tau=1.0)
    bad_mode.mode = 7
    assert _dr(L, bad_mode) == nabla.ERR_PARAM
    assert _dr(L, thr(tau=1.0), q=None) == nabla.ERR_NULL         # the threshold mode reads q, k
    assert _dr(L, thr(tau=1.0), k=FAKE_ODD) == nabla.ERR_ALIGN
    assert _dr(L, thr(tau=1.0), ws_bytes=1024) == nabla.ERR_WORKSPACE
    # the static mode reads neither q nor k and needs only the status region
    assert _dr(L, ratio(gamma=0.5), q=None, k=None, ws_bytes=16) == nabla.ERR_WORKSPACE
    assert _dr(L, ratio(gamma=0.5), shape=_shape(P=4)) == nabla.ERR_SHAPE
    assert L.nabla_build_mask_dr(ctypes.byref(_shape()), None, FAKE, FAKE, ctypes.byref(_mask()),
                                 FAKE, 1 << 40, None) == nabla.ERR_NULL


def test_attention_rejects_on_host(L):
    s, good = _shape(), nabla.params_of(0.7, (3, 3, 3), D=128)
    m = _mask()
    fwd = lambda *a: L.nabla_attn_fwd(ctypes.byref(s), ctypes.byref(good), *a)
    assert fwd(FAKE, FAKE, None, ctypes.byref(m), FAKE, None, FAKE, 1 << 40, None) == nabla.ERR_NULL
    assert fwd(FAKE, FAKE_ODD, FAKE, ctypes.byref(m), FAKE, None, FAKE, 1 << 40, None) == \
        nabla.ERR_ALIGN
    assert fwd(FAKE, FAKE, FAKE, ctypes.byref(m), FAKE, None, FAKE, 16, None) == \
        nabla.ERR_WORKSPACE
    nocols = nabla.MaskStruct(FAKE, FAKE, FAKE, None, None)
    bwd = lambda mask, ws_bytes: L.nabla_attn_bwd(
        ctypes.byref(s), ctypes.byref(good), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
        ctypes.byref(mask), FAKE, FAKE, FAKE, FAKE, ws_bytes, None)
    assert bwd(nocols, 1 << 40) == nabla.ERR_NULL  # backward needs column lists
    assert bwd(m, 1024) == nabla.ERR_WORKSPACE


def test_flatten_rejects_on_host(L):
    f = L.nabla_flatten
    assert f(None, FAKE, 1, 2, 16, 16, 8, 256, 0, None) == nabla.ERR_NULL
    assert f(None, None, 0, 2, 16, 16, 8, 256, 0, None) == nabla.OK  # empty: nothing to touch
    assert f(FAKE, FAKE_ODD, 1, 2, 16, 16, 8, 256, 0, None) == nabla.ERR_ALIGN
    assert f(FAKE, ctypes.c_void_p(0x20000), 1, 2, 16, 16, 8, 24, 0, None) == nabla.ERR_ALIGN
    assert f(FAKE, ctypes.c_void_p(0x20000), 1, 2, 16, 12, 8, 256, 0, None) == nabla.ERR_SHAPE
    assert f(FAKE, FAKE, 1, 2, 16, 16, 8, 256, 0, None) == nabla.ERR_PARAM  # in place
    # partially overlapping buffers (out starts inside in)
    assert f(FAKE, ctypes.c_void_p(0x10000 + 4096), 1, 2, 16, 16, 8, 256, 0, None) == \
        nabla.ERR_PARAM
    # empty inputs are a successful no-op
    assert f(FAKE, ctypes.c_void_p(0x20000), 0, 2, 16, 16, 8, 256, 0, None) == nabla.OK


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(nabla, "_lib", None)
    monkeypatch.setattr(nabla, "LIB_PATH", "/nonexistent/libnabla.so")
    with pytest.raises(RuntimeError, match="not built"):
        nabla.lib()

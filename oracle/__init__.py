"""CPU oracle for NABLA block-sparse attention -- TEST INFRASTRUCTURE ONLY.

Plain, slow, explicit-loop restatement of the method described in "NABLA:
Neighborhood Adaptive Block-Level Attention" (technical summary, section
"手法: NABLA"), in float64 with the mask decision also available in the
precision the GPU kernels take it in (see nabla_oracle.c).  Only the tests,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package.  It shares no code with the CUDA library and never imports it.

All arrays are numpy.  bf16 tensors are passed as their raw uint16 bits.
"""
import ctypes
import os

import numpy as np

from .build import build as _build

NO_STA = 1
FULL_STA = 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_D = ctypes.c_double
_F = ctypes.c_float
_U = ctypes.c_uint


def _declare(L):
    L.oracle_flat_index.restype = _I64
    L.oracle_flat_index.argtypes = [_I] * 7
    L.oracle_flatten.restype = None
    L.oracle_flatten.argtypes = [_P, _P, _I64, _I, _I, _I, _I, _I64, _I]
    L.oracle_pool_f64.restype = None
    L.oracle_pool_f64.argtypes = [_P, _P, _I64, _I64, _I, _I]
    L.oracle_pool_f32.restype = None
    L.oracle_pool_f32.argtypes = [_P, _P, _I64, _I64, _I, _I]
    L.oracle_sta.restype = _I
    L.oracle_sta.argtypes = [_I64, _I64, _I, _I, _I, _I, _I, _U]
    L.oracle_mask_f64.restype = None
    L.oracle_mask_f64.argtypes = [_P, _P, _I64, _I64, _I, _I, _I, _D, _D, _I, _I, _I, _U,
                                  _P, _P, _P, _P, _P, _P, _P, _P]
    L.oracle_scores_f32.restype = None
    L.oracle_scores_f32.argtypes = [_P, _P, _I64, _I64, _I, _F, _P]
    L.oracle_mask_from_scores.restype = None
    L.oracle_mask_from_scores.argtypes = [_P, _I64, _I64, _I, _I, _F, _I, _I, _I, _U,
                                          _P, _P, _P, _P, _P, _P, _P]
    L.oracle_mask.restype = None
    L.oracle_mask.argtypes = [_P, _P, _I64, _I64, _I, _I, _I, _F, _F, _I, _I, _I, _U,
                              _P, _P, _P, _P, _P, _P, _P]
    L.oracle_dr_static.restype = None
    L.oracle_dr_static.argtypes = [_I64, _I64, _I, _I, _I, _D, _D, _I, _I, _I, _U,
                                   _P, _P, _P, _P, _P, _P]
    L.oracle_dr_threshold.restype = None
    L.oracle_dr_threshold.argtypes = [_P, _P, _I64, _I64, _I, _I, _I, _F, _F, _I, _I, _I, _U,
                                      _P, _P, _P, _P, _P, _P]
    L.oracle_cut_row_f64.restype = _I64
    L.oracle_cut_row_f64.argtypes = [_P, _I64, _D, _P]
    L.oracle_cut_row_fixed.restype = _I64
    L.oracle_cut_row_fixed.argtypes = [_P, _I64, _F, _P]
    L.oracle_attn_fwd.restype = None
    L.oracle_attn_fwd.argtypes = [_P, _P, _P, _I64, _I64, _I, _I, _P, _P, _D, _P, _P, _I64,
                                  _P, _P]
    L.oracle_attn_bwd.restype = None
    L.oracle_attn_bwd.argtypes = [_P, _P, _P, _P, _I64, _I64, _I, _I, _P, _P, _P, _P, _D,
                                  _P, _P, _I64, _P, _P, _I64, _P, _P, _P]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# Fractal flattening
# --------------------------------------------------------------------------

def flat_index(t, y, x, T, H, W, P):
    return int(lib().oracle_flat_index(t, y, x, T, H, W, P))


def permutation(T, H, W, P):
    """perm[n_grid] = n_flat for the row-major grid index n_grid."""
    out = np.empty(T * H * W, dtype=np.int64)
    n = 0
    for t in range(T):
        for y in range(H):
            for x in range(W):
                out[n] = flat_index(t, y, x, T, H, W, P)
                n += 1
    return out


def flatten(x, T, H, W, P, inverse=False):
    """x: array whose leading dims are [outer..., T*H*W or T,H,W, inner...]
    given as a contiguous byte buffer shaped [outer, T*H*W, inner_bytes]."""
    x = np.ascontiguousarray(x)
    outer = x.shape[0]
    inner_bytes = x.nbytes // (outer * T * H * W)
    out = np.empty_like(x)
    lib().oracle_flatten(_ptr(x), _ptr(out), outer, T, H, W, P, inner_bytes, int(inverse))
    return out


def flatten_tokens(x_bits, T, H, W, P, inverse=False):
    """[BH, N, D] uint16 (bf16 bits) in grid order -> flattened order
    (or back with inverse=True)."""
    x_bits = _c(x_bits, np.uint16)
    BH, N, D = x_bits.shape
    f = flatten(x_bits.view(np.uint8).reshape(BH, N, 2 * D), T, H, W, P, inverse)
    return f.view(np.uint16).reshape(BH, N, D)


# --------------------------------------------------------------------------
# Pooling, scores, masks
# --------------------------------------------------------------------------

def pool_f64(x_bits, L=64):
    x_bits = _c(x_bits, np.uint16)
    BH, N, D = x_bits.shape
    out = np.empty((BH, N // L, D), dtype=np.float64)
    lib().oracle_pool_f64(_ptr(x_bits), _ptr(out), BH, N, D, L)
    return out


def pool_f32(x_bits, L=64):
    x_bits = _c(x_bits, np.uint16)
    BH, N, D = x_bits.shape
    out = np.empty((BH, N // L, D), dtype=np.float32)
    lib().oracle_pool_f32(_ptr(x_bits), _ptr(out), BH, N, D, L)
    return out


def sta(i, j, Hp, Wp, window, flags=0):
    wt, wh, ww = window
    return bool(lib().oracle_sta(i, j, Hp, Wp, wt, wh, ww, flags))


def scores_f32(qbar, kbar, scale):
    qbar = _c(qbar, np.float32)
    kbar = _c(kbar, np.float32)
    BH, nb, D = qbar.shape
    out = np.empty((BH, nb, nb), dtype=np.float32)
    lib().oracle_scores_f32(_ptr(qbar), _ptr(kbar), BH, nb, D, np.float32(scale), _ptr(out))
    return out


def _mask_buffers(BH, nb, cols):
    words = (nb + 31) // 32
    m = dict(bits=np.zeros((BH, nb, words), dtype=np.uint32),
             row_idx=np.zeros((BH, nb, nb), dtype=np.uint16),
             row_cnt=np.zeros((BH, nb), dtype=np.int32),
             adapt_cnt=np.zeros((BH, nb), dtype=np.int32))
    if cols:
        m["col_idx"] = np.zeros((BH, nb, nb), dtype=np.uint16)
        m["col_cnt"] = np.zeros((BH, nb), dtype=np.int32)
    return m


def mask(qbar, kbar, grid, p, scale, window=(3, 3, 3), flags=0, cols=True):
    """Mask in the GPU's decision precision from float32 pooled means.
    grid = (T, Hp, Wp) in blocks.  Returns a dict of arrays (see C header)."""
    qbar = _c(qbar, np.float32)
    kbar = _c(kbar, np.float32)
    BH, nb, D = qbar.shape
    T, Hp, Wp = grid
    assert T * Hp * Wp == nb
    m = _mask_buffers(BH, nb, cols)
    m["margin"] = np.zeros((BH, nb), dtype=np.float64)
    lib().oracle_mask(_ptr(qbar), _ptr(kbar), BH, nb, D, Hp, Wp, np.float32(p),
                      np.float32(scale), *window, flags, _ptr(m["bits"]), _ptr(m["row_idx"]),
                      _ptr(m["row_cnt"]), _ptr(m.get("col_idx")), _ptr(m.get("col_cnt")),
                      _ptr(m["adapt_cnt"]), _ptr(m["margin"]))
    return m


def mask_from_scores(scores, grid, p, window=(3, 3, 3), flags=0, cols=True):
    """Mask in decision precision from given float32 score rows [BH, nb, nb]
    (for instance the scores a kernel reports): the same cut, STA and
    diagonal as mask(), applied to those values."""
    scores = _c(scores, np.float32)
    BH, nb, nb2 = scores.shape
    assert nb == nb2
    T, Hp, Wp = grid
    assert T * Hp * Wp == nb
    m = _mask_buffers(BH, nb, cols)
    m["margin"] = np.zeros((BH, nb), dtype=np.float64)
    lib().oracle_mask_from_scores(_ptr(scores), BH, nb, Hp, Wp, np.float32(p), *window, flags,
                                  _ptr(m["bits"]), _ptr(m["row_idx"]), _ptr(m["row_cnt"]),
                                  _ptr(m.get("col_idx")), _ptr(m.get("col_cnt")),
                                  _ptr(m["adapt_cnt"]), _ptr(m["margin"]))
    return m


def mask_f64(qbar, kbar, grid, p, scale, window=(3, 3, 3), flags=0, cols=True):
    """Plain float64 mask from float64 pooled means."""
    qbar = _c(qbar, np.float64)
    kbar = _c(kbar, np.float64)
    BH, nb, D = qbar.shape
    T, Hp, Wp = grid
    assert T * Hp * Wp == nb
    m = _mask_buffers(BH, nb, cols)
    m["cum_before"] = np.zeros((BH, nb), dtype=np.float64)
    m["cum_at"] = np.zeros((BH, nb), dtype=np.float64)
    lib().oracle_mask_f64(_ptr(qbar), _ptr(kbar), BH, nb, D, Hp, Wp, float(p), float(scale),
                          *window, flags, _ptr(m["bits"]), _ptr(m["row_idx"]),
                          _ptr(m["row_cnt"]), _ptr(m.get("col_idx")), _ptr(m.get("col_cnt")),
                          _ptr(m["adapt_cnt"]), _ptr(m["cum_before"]), _ptr(m["cum_at"]))
    return m


def dr_static(BH, grid, gamma, lam, window=(3, 3, 3), flags=0, cols=True):
    """DynamicRad static-ratio mask (content-free) for BH heads of a grid
    (T, Hp, Wp) in blocks."""
    T, Hp, Wp = grid
    nb = T * Hp * Wp
    m = _mask_buffers(BH, nb, cols)
    lib().oracle_dr_static(BH, nb, T, Hp, Wp, float(gamma), float(lam), *window, flags,
                           _ptr(m["bits"]), _ptr(m["row_idx"]), _ptr(m["row_cnt"]),
                           _ptr(m.get("col_idx")), _ptr(m.get("col_cnt")), _ptr(m["adapt_cnt"]))
    return m


def dr_threshold(qbar, kbar, grid, tau, scale, window=(3, 3, 3), flags=0, cols=True):
    """DynamicRad logit-threshold mask from float32 pooled means."""
    qbar = _c(qbar, np.float32)
    kbar = _c(kbar, np.float32)
    BH, nb, D = qbar.shape
    T, Hp, Wp = grid
    assert T * Hp * Wp == nb
    m = _mask_buffers(BH, nb, cols)
    lib().oracle_dr_threshold(_ptr(qbar), _ptr(kbar), BH, nb, D, Hp, Wp, np.float32(tau),
                              np.float32(scale), *window, flags, _ptr(m["bits"]),
                              _ptr(m["row_idx"]), _ptr(m["row_cnt"]), _ptr(m.get("col_idx")),
                              _ptr(m.get("col_cnt")), _ptr(m["adapt_cnt"]))
    return m


def cut_row_f64(score, p):
    score = _c(score, np.float64)
    keep = np.zeros(score.shape[0], dtype=np.uint8)
    lib().oracle_cut_row_f64(_ptr(score), score.shape[0], float(p), _ptr(keep))
    return keep.astype(bool)


def cut_row_fixed(score, p):
    score = _c(score, np.float32)
    keep = np.zeros(score.shape[0], dtype=np.uint8)
    lib().oracle_cut_row_fixed(_ptr(score), score.shape[0], np.float32(p), _ptr(keep))
    return keep.astype(bool)


def build_mask(q_bits, k_bits, grid, p, scale, window=(3, 3, 3), flags=0, cols=True):
    """The whole decision path from flattened bf16 Q and K bits [BH, N, D]."""
    return mask(pool_f32(q_bits), pool_f32(k_bits), grid, p, scale, window, flags, cols)


def lists_to_dense(row_idx, row_cnt):
    """Block mask as a boolean [BH, nb, nb] array from row lists."""
    BH, nb = row_cnt.shape
    out = np.zeros((BH, nb, nb), dtype=bool)
    for bh in range(BH):
        for i in range(nb):
            out[bh, i, row_idx[bh, i, :row_cnt[bh, i]]] = True
    return out


# --------------------------------------------------------------------------
# Attention (float64)
# --------------------------------------------------------------------------

def bf16_bits_to_f64(bits):
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _sel(sel):
    if sel is None:
        return None, None, 0
    sel = np.asarray(sel, dtype=np.int64).reshape(-1, 2)
    return np.ascontiguousarray(sel[:, 0]), np.ascontiguousarray(sel[:, 1]), sel.shape[0]


def attn_fwd(q, k, v, row_idx, row_cnt, scale, sel=None, L=64):
    """q, k, v: float64 [BH, N, D] flattened.  sel: list of (bh, i) query
    blocks or None for all.  Returns (o [n_sel, L, D], lse [n_sel, L])."""
    q, k, v = (_c(a, np.float64) for a in (q, k, v))
    BH, N, D = q.shape
    row_idx = _c(row_idx, np.uint16)
    row_cnt = _c(row_cnt, np.int32)
    sb, si, ns = _sel(sel)
    if sel is None:
        ns = BH * (N // L)
    o = np.empty((ns, L, D), dtype=np.float64)
    lse = np.empty((ns, L), dtype=np.float64)
    lib().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), BH, N, D, L, _ptr(row_idx), _ptr(row_cnt),
                          float(scale), _ptr(sb), _ptr(si), ns, _ptr(o), _ptr(lse))
    return o, lse


def attn_bwd(q, k, v, dout, row_idx, row_cnt, col_idx, col_cnt, scale, dq_sel=None,
             kv_sel=None, L=64):
    """Gradients of the block-sparse attention.  Returns (dq [n_dq, L, D],
    dk [n_kv, L, D], dv [n_kv, L, D]) for the selected blocks (None = all)."""
    q, k, v, dout = (_c(a, np.float64) for a in (q, k, v, dout))
    BH, N, D = q.shape
    row_idx = _c(row_idx, np.uint16)
    row_cnt = _c(row_cnt, np.int32)
    col_idx = _c(col_idx, np.uint16)
    col_cnt = _c(col_cnt, np.int32)
    qb, qi, nq = _sel(dq_sel)
    kb, kj, nk = _sel(kv_sel)
    if dq_sel is None:
        nq = BH * (N // L)
    if kv_sel is None:
        nk = BH * (N // L)
    dq = np.empty((nq, L, D), dtype=np.float64)
    dk = np.empty((nk, L, D), dtype=np.float64)
    dv = np.empty((nk, L, D), dtype=np.float64)
    lib().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), BH, N, D, L, _ptr(row_idx),
                          _ptr(row_cnt), _ptr(col_idx), _ptr(col_cnt), float(scale), _ptr(qb),
                          _ptr(qi), nq, _ptr(kb), _ptr(kj), nk, _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv

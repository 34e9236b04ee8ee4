"""Thin ctypes binding of libnabla.so (include/nabla.h).

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every step runs in the library's kernels.  There is no
fallback: if the library is missing or a call fails, this module raises.
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnabla.so")

OK = 0
ERR_SHAPE, ERR_ALIGN, ERR_PARAM, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_NULL = (
    -1, -2, -3, -4, -5, -6, -7)
NO_STA, FULL_STA, EMIT_COLS, DEBUG_SCORES, DEBUG_TIMEOUT = 1, 2, 4, 8, 0x100
OP_BUILD_MASK, OP_ATTN_FWD, OP_ATTN_BWD = 0, 1, 2
MASK_BITS, MASK_ROW_IDX, MASK_ROW_CNT, MASK_COL_IDX, MASK_COL_CNT, MASK_SCORES = 0, 1, 2, 3, 4, 5

# every symbol include/nabla.h declares
SYMBOLS = ("nabla_flatten", "nabla_workspace_size", "nabla_mask_bytes", "nabla_build_mask",
           "nabla_build_mask_grid", "nabla_build_mask_static", "nabla_build_mask_dr",
           "nabla_attn_fwd", "nabla_attn_bwd", "nabla_status", "nabla_strerror")
DR_STATIC_RATIO, DR_THRESHOLD = 0, 1


class NablaError(RuntimeError):
    def __init__(self, status, what):
        super().__init__("%s failed: %s (%d)" % (what, strerror(status), status))
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "heads", "T", "H", "W", "D", "P")]


class Params(ctypes.Structure):
    _fields_ = [("p", ctypes.c_float), ("sta_t", ctypes.c_int), ("sta_h", ctypes.c_int),
                ("sta_w", ctypes.c_int), ("scale", ctypes.c_float), ("flags", ctypes.c_uint)]


class DrParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("gamma", ctypes.c_double), ("lambda_", ctypes.c_double),
                ("tau", ctypes.c_float), ("sta_t", ctypes.c_int), ("sta_h", ctypes.c_int),
                ("sta_w", ctypes.c_int), ("scale", ctypes.c_float), ("flags", ctypes.c_uint)]


class MaskStruct(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p)
                for n in ("bits", "row_idx", "row_cnt", "col_idx", "col_cnt", "scores")]


_lib = None


def lib():
    """Load libnabla.so; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libnabla.so is not built; run "
                               "`python -m adaptive_block_sparse_fractal_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.nabla_flatten.argtypes = [P, P, I64, I, I, I, I, I64, I, P]
        L.nabla_flatten.restype = I
        L.nabla_workspace_size.argtypes = [P, I]
        L.nabla_workspace_size.restype = SZ
        L.nabla_mask_bytes.argtypes = [P, I]
        L.nabla_mask_bytes.restype = SZ
        L.nabla_build_mask.argtypes = [P, P, P, P, P, P, SZ, P]
        L.nabla_build_mask.restype = I
        L.nabla_build_mask_grid.argtypes = [P, P, P, P, P, P, P, P, SZ, P]
        L.nabla_build_mask_grid.restype = I
        L.nabla_build_mask_static.argtypes = [P, P, P, P, P, P]
        L.nabla_build_mask_static.restype = I
        L.nabla_build_mask_dr.argtypes = [P, P, P, P, P, P, SZ, P]
        L.nabla_build_mask_dr.restype = I
        L.nabla_attn_fwd.argtypes = [P, P, P, P, P, P, P, P, P, SZ, P]
        L.nabla_attn_fwd.restype = I
        L.nabla_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.nabla_attn_bwd.restype = I
        L.nabla_status.argtypes = [P, P]
        L.nabla_status.restype = I
        L.nabla_strerror.argtypes = [I]
        L.nabla_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


def strerror(status):
    return lib().nabla_strerror(int(status)).decode()


def _check(status, what):
    if status != OK:
        raise NablaError(status, what)


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError("%s must be a contiguous CUDA %s tensor" % (name, dtype))


def shape_of(B, heads, T, H, W, D, P=8):
    return Shape(B, heads, T, H, W, D, P)


def params_of(p, window=(3, 3, 3), scale=None, D=None, flags=0):
    if scale is None:
        scale = D ** -0.5
    return Params(float(p), int(window[0]), int(window[1]), int(window[2]), float(scale),
                  int(flags))


def dr_params_of(mode, gamma=1.0, lam=0.0, tau=0.0, window=(3, 3, 3), scale=None, D=None,
                 flags=0):
    if scale is None:
        scale = D ** -0.5
    return DrParams(int(mode), float(gamma), float(lam), float(tau), int(window[0]),
                    int(window[1]), int(window[2]), float(scale), int(flags))


def workspace_size(shape, op):
    return int(lib().nabla_workspace_size(ctypes.byref(shape), op))


def mask_bytes(shape, part):
    return int(lib().nabla_mask_bytes(ctypes.byref(shape), part))


def workspace(shape, op, device):
    n = workspace_size(shape, op)
    if n == 0:
        raise NablaError(ERR_SHAPE, "workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def alloc_mask(shape, device, cols=True, scores=False):
    BH, nb = shape.B * shape.heads, shape.T * (shape.H // shape.P) * (shape.W // shape.P)
    words = (nb + 31) // 32
    m = {"bits": torch.empty((BH, nb, words), dtype=torch.int32, device=device),
         "row_idx": torch.empty((BH, nb, nb), dtype=torch.int16, device=device),
         "row_cnt": torch.empty((BH, nb), dtype=torch.int32, device=device)}
    if cols:
        m["col_idx"] = torch.empty((BH, nb, nb), dtype=torch.int16, device=device)
        m["col_cnt"] = torch.empty((BH, nb), dtype=torch.int32, device=device)
    if scores:
        m["scores"] = torch.empty((BH, nb, nb), dtype=torch.float32, device=device)
    for part, key in ((MASK_BITS, "bits"), (MASK_ROW_IDX, "row_idx"), (MASK_ROW_CNT, "row_cnt"),
                      (MASK_COL_IDX, "col_idx"), (MASK_COL_CNT, "col_cnt"),
                      (MASK_SCORES, "scores")):
        if key in m:
            assert m[key].numel() * m[key].element_size() == mask_bytes(shape, part)
    return m


def _mask_struct(m):
    return MaskStruct(*(_ptr(m.get(k)) for k in ("bits", "row_idx", "row_cnt", "col_idx",
                                                  "col_cnt", "scores")))


def flatten(x, T, H, W, P=8, inverse=False, out=None):
    """x: contiguous CUDA tensor whose bytes are [outer, T*H*W, inner] in grid
    order (inverse=False) or flattened order (inverse=True); dim 0 is outer."""
    if not (x.is_cuda and x.is_contiguous()):
        raise ValueError("x must be a contiguous CUDA tensor")
    out = torch.empty_like(x) if out is None else out
    outer = x.shape[0]
    total = x.numel() * x.element_size()
    inner = total // (outer * T * H * W) if outer else 0
    _check(lib().nabla_flatten(_ptr(x), _ptr(out), outer, T, H, W, P, inner, int(inverse),
                               _stream(x)), "nabla_flatten")
    return out


def build_mask(shape, params, q, k, mask=None, ws=None):
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    cols = bool(params.flags & EMIT_COLS)
    dbg = bool(params.flags & DEBUG_SCORES)
    mask = alloc_mask(shape, q.device, cols, dbg) if mask is None else mask
    ws = workspace(shape, OP_BUILD_MASK, q.device) if ws is None else ws
    ms = _mask_struct(mask)
    _check(lib().nabla_build_mask(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k),
                                  ctypes.byref(ms), _ptr(ws), ws.numel(), _stream(q)),
           "nabla_build_mask")
    return mask


def build_mask_dr(shape, params, q=None, k=None, mask=None, ws=None, device=None):
    """DynamicRad-style mask (static ratio or logit threshold) in the same
    format; q and k are needed by the threshold mode only."""
    thr = params.mode == DR_THRESHOLD
    if thr:
        _need(q, torch.bfloat16, "q")
        _need(k, torch.bfloat16, "k")
        device = q.device
    cols = bool(params.flags & EMIT_COLS)
    dbg = bool(params.flags & DEBUG_SCORES)
    mask = alloc_mask(shape, device, cols, dbg) if mask is None else mask
    if ws is None:
        ws = workspace(shape, OP_BUILD_MASK if thr else OP_ATTN_FWD, device)
    ms = _mask_struct(mask)
    stream = ctypes.c_void_p(torch.cuda.current_stream(ws.device).cuda_stream)
    _check(lib().nabla_build_mask_dr(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k),
                                     ctypes.byref(ms), _ptr(ws), ws.numel(), stream),
           "nabla_build_mask_dr")
    return mask


def build_mask_grid(shape, params, q_grid, k_grid, q=None, k=None, mask=None, ws=None):
    """Flatten q_grid, k_grid (grid order, any shape holding [B*h, T*H*W, D])
    into q, k and build the mask from them in one call; returns (q, k, mask)."""
    _need(q_grid, torch.bfloat16, "q_grid")
    _need(k_grid, torch.bfloat16, "k_grid")
    q = torch.empty_like(q_grid) if q is None else q
    k = torch.empty_like(k_grid) if k is None else k
    cols = bool(params.flags & EMIT_COLS)
    dbg = bool(params.flags & DEBUG_SCORES)
    mask = alloc_mask(shape, q_grid.device, cols, dbg) if mask is None else mask
    ws = workspace(shape, OP_BUILD_MASK, q_grid.device) if ws is None else ws
    ms = _mask_struct(mask)
    _check(lib().nabla_build_mask_grid(ctypes.byref(shape), ctypes.byref(params), _ptr(q_grid),
                                       _ptr(k_grid), _ptr(q), _ptr(k), ctypes.byref(ms), _ptr(ws),
                                       ws.numel(), _stream(q_grid)), "nabla_build_mask_grid")
    return q, k, mask


def attn_fwd(shape, params, q, k, v, mask, o=None, lse=None, ws=None, want_lse=True):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    o = torch.empty_like(q) if o is None else o
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    ws = workspace(shape, OP_ATTN_FWD, q.device) if ws is None else ws
    ms = _mask_struct(mask)
    _check(lib().nabla_attn_fwd(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k),
                                _ptr(v), ctypes.byref(ms), _ptr(o), _ptr(lse), _ptr(ws),
                                ws.numel(), _stream(q)), "nabla_attn_fwd")
    return o, lse


def attn_bwd(shape, params, q, k, v, o, dout, lse, mask, dq=None, dk=None, dv=None, ws=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, torch.bfloat16, n)
    _need(lse, torch.float32, "lse")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = workspace(shape, OP_ATTN_BWD, q.device) if ws is None else ws
    ms = _mask_struct(mask)
    _check(lib().nabla_attn_bwd(ctypes.byref(shape), ctypes.byref(params), _ptr(q), _ptr(k),
                                _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), ctypes.byref(ms),
                                _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), _stream(q)),
           "nabla_attn_bwd")
    return dq, dk, dv


def status(ws):
    """Synchronise the current stream and return the workspace status word."""
    return int(lib().nabla_status(_ptr(ws), _stream(ws)))

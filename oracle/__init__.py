"""ctypes front end of the CPU oracle (oracle/rat_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by
bench.py's CPU-baseline leg.  The product path (the CUDA library and its Python
binding) never imports this package, and this package imports nothing from the
product.

All arrays are numpy float64 in the operator's row-major layouts:
  x, g, q, k, v, o : [B, T, H, d]     init, final : [B, H, d]
"""
import ctypes
import os

import numpy as np

from .build import build as build_library

_lib = None


def _load():
    global _lib
    if _lib is None:
        # RAT_ORACLE_LIB points at another build of rat_oracle.c (the mutation
        # test loads deliberately broken copies through it).
        path = os.environ.get("RAT_ORACLE_LIB") or build_library()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        up = ctypes.POINTER(ctypes.c_ubyte)
        lp = ctypes.POINTER(ctypes.c_int64)
        lib.oracle_scan.argtypes = [ctypes.c_int] * 4 + [dp, dp, dp, up, dp, dp]
        lib.oracle_scan.restype = None
        lib.oracle_attn_rows.argtypes = [ctypes.c_int] * 4 + [dp, dp, dp, ip, ip, ctypes.c_double,
                                                              ctypes.c_int, ctypes.c_long, lp, dp, dp]
        lib.oracle_attn_rows.restype = ctypes.c_int
        lib.oracle_attn_rows_grid.argtypes = lib.oracle_attn_rows.argtypes
        lib.oracle_attn_rows_grid.restype = ctypes.c_int
        lib.oracle_attn_rows_ex.argtypes = lib.oracle_attn_rows.argtypes + [ctypes.c_int, ctypes.c_int]
        lib.oracle_attn_rows_ex.restype = ctypes.c_int
        lib.oracle_attn_rows_topk.argtypes = [ctypes.c_int] * 4 + [dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                                                  ctypes.c_int, ctypes.c_double, ctypes.c_long,
                                                                  lp, dp, dp]
        lib.oracle_attn_rows_topk.restype = ctypes.c_int
        lib.oracle_topk_select.argtypes = [ctypes.c_int] * 4 + [dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                              ctypes.c_long, lp, ctypes.POINTER(ctypes.c_int), dp]
        lib.oracle_topk_select.restype = ctypes.c_int
        lib.oracle_decode_step.argtypes = [ctypes.c_int] * 4 + [ip, dp, dp, dp, dp, ip, ip, up,
                                                                ctypes.c_double, dp, dp, dp, dp, dp, dp]
        lib.oracle_decode_step.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dp(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _u8(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.uint8)


def default_scale(d: int) -> float:
    return 1.0 / np.sqrt(d)


def scan(x, g, init=None, recur=None):
    """Gated linear recurrence per channel; returns (out [B,T,H,d], final [B,H,d])."""
    lib = _load()
    x, g, init, recur = _f64(x), _f64(g), _f64(init), _u8(recur)
    B, T, H, d = x.shape
    assert g.shape == x.shape
    out = np.empty_like(x)
    final = np.empty((B, H, d), dtype=np.float64)
    lib.oracle_scan(B, T, H, d, _dp(x), _dp(g), _dp(init),
                    None if recur is None else recur.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)),
                    _dp(out), _dp(final))
    return out, final


def attn_rows(q, kt, vt, dil, win, rows, parts=3, scale=None, grid=False, dedupe=False):
    """Rows (b, h, t) of the attention step; returns (o [n,d], lse [n]).
    grid=True takes the fixed-grid reading of the dilated part (keys j <= t
    with j mod D == D - 1, plus t) instead of the residue set; dedupe=True
    counts a key that both parts hold once (the window part skips it)."""
    lib = _load()
    q, kt, vt = _f64(q), _f64(kt), _f64(vt)
    B, T, H, d = q.shape
    dil, win = _i32(dil), _i32(win)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    s = default_scale(d) if scale is None else float(scale)
    rc = lib.oracle_attn_rows_ex(B, T, H, d, _dp(q), _dp(kt), _dp(vt),
                                 dil.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                 win.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), s, int(parts), n,
                                 rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), _dp(o), _dp(lse),
                                 int(bool(grid)), int(bool(dedupe)))
    if rc != 0:
        raise ValueError("oracle_attn_rows: invalid arguments")
    return o, lse


def attn_rows_topk(q, kt, vt, block, K, mode, rows, scale=None):
    """Rows (b, h, t) of top-k block attention (mode "quest": per-channel
    min/max block statistics; "moba": mean-pooled block keys); returns
    (o [n,d], lse [n])."""
    lib = _load()
    q, kt, vt = _f64(q), _f64(kt), _f64(vt)
    B, T, H, d = q.shape
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    s = default_scale(d) if scale is None else float(scale)
    m = {"quest": 0, "moba": 1}[mode]
    rc = lib.oracle_attn_rows_topk(B, T, H, d, _dp(q), _dp(kt), _dp(vt), int(block), int(K), m, s, n,
                                   rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), _dp(o), _dp(lse))
    if rc != 0:
        raise ValueError("oracle_attn_rows_topk: invalid arguments")
    return o, lse


def topk_select(q, kt, block, K, mode, rows):
    """The block selection of attn_rows_topk for each row: (sel [n, K] int32 in
    pick order, -1 padded; gap [n]: last pick's score minus the best score
    left out, +inf when nothing is left out)."""
    lib = _load()
    q, kt = _f64(q), _f64(kt)
    B, T, H, d = q.shape
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    sel = np.empty((n, max(int(K), 1)), dtype=np.int32)
    gap = np.empty((n,), dtype=np.float64)
    m = {"quest": 0, "moba": 1}[mode]
    rc = lib.oracle_topk_select(B, T, H, d, _dp(q), _dp(kt), int(block), int(K), m, n,
                                rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                sel.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), _dp(gap))
    if rc != 0:
        raise ValueError("oracle_topk_select: invalid arguments")
    return sel[:, :K], gap


def all_rows(B, T, H):
    """Every (b, h, t) triple in (b, h, t) order."""
    b, h, t = np.meshgrid(np.arange(B), np.arange(H), np.arange(T), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), t.ravel()], axis=1)


def attention(q, kt, vt, dil, win, parts=3, scale=None, grid=False, dedupe=False):
    """Every row of the attention step as full tensors: (o [B,T,H,d], lse [B,H,T])."""
    B, T, H, d = q.shape
    rows = all_rows(B, T, H)
    o, lse = attn_rows(q, kt, vt, dil, win, rows, parts=parts, scale=scale, grid=grid, dedupe=dedupe)
    o = o.reshape(B, H, T, d).transpose(0, 2, 1, 3).copy()
    return o, lse.reshape(B, H, T)


def mix_prefill(q, k, v, g, dil, win, recur, init_k=None, init_v=None, scale=None):
    """The whole operator for a prefill: scan of k and v, then attention."""
    kt, fk = scan(k, g, init_k, recur)
    vt, fv = scan(v, g, init_v, recur)
    o, lse = attention(q, kt, vt, dil, win, parts=3, scale=scale)
    return dict(o=o, lse=lse, kt=kt, vt=vt, final_k=fk, final_v=fv)


def decode_step(q, k, v, g, state_k, state_v, hist_k, hist_v, pos, dil, win, recur, scale=None):
    """One decode step.  q,k,v,g,state_*: [B,H,d]; hist_*: [B,cap,H,d] natural order.
    state_* and hist_* are updated in place (they must be float64 contiguous arrays).
    Returns (o [B,H,d], lse [B,H])."""
    lib = _load()
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    for a in (state_k, state_v, hist_k, hist_v):
        assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    B, H, d = q.shape
    cap = hist_k.shape[1]
    pos = _i32(pos)
    dil, win = _i32(dil), _i32(win)
    recur = _u8(recur)
    o = np.empty((B, H, d), dtype=np.float64)
    lse = np.empty((B, H), dtype=np.float64)
    s = default_scale(d) if scale is None else float(scale)
    ip = ctypes.POINTER(ctypes.c_int)
    rc = lib.oracle_decode_step(B, H, d, cap, pos.ctypes.data_as(ip), _dp(q), _dp(k), _dp(v), _dp(g),
                                dil.ctypes.data_as(ip), win.ctypes.data_as(ip),
                                None if recur is None else recur.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)),
                                s, _dp(state_k), _dp(state_v), _dp(hist_k), _dp(hist_v), _dp(o), _dp(lse))
    if rc != 0:
        raise ValueError("oracle_decode_step: invalid arguments")
    return o, lse

"""Python binding of librat.so, the sm_100a implementation of the RAT+
temporal-mixing operator ("RAT+: Train Dense, Infer Sparse -- Recurrence
Augmented Attention for Dilated Inference": Figure 1(a)/(c), Figure 2).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  Each function has the name and argument order of the C entry
point in include/rat.h and takes torch tensors for the device buffers (torch is
used for device memory and streams).  There is no fallback: importing works
without a GPU (so the symbols can be inspected), but every compute call raises
if the library is missing or the tensors are not on a CUDA device.
"""
import ctypes
import os

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librat.so")

RAT_OK, RAT_ERR_INVALID, RAT_ERR_UNSUPPORTED, RAT_ERR_CUDA, RAT_ERR_TIMEOUT, RAT_ERR_WORKSPACE = range(6)
RAT_F32, RAT_BF16 = 0, 1
RAT_OP_SCAN, RAT_OP_ATTN, RAT_OP_MIX, RAT_OP_MIX_CALLER_KV, RAT_OP_DECODE, RAT_OP_TOPK_DECODE = range(6)
RAT_TOPK_QUEST, RAT_TOPK_MOBA = 0, 1
RAT_FLAG_GRID_DILATION = 1
RAT_FLAG_DEDUPE = 2
RAT_FLAG_SEPARATE_GATES = 4

EXPORTS = ["rat_workspace_size", "rat_workspace_init", "rat_cache_rows", "rat_scan_prefill",
           "rat_dilated_attn_prefill", "rat_mix_prefill", "rat_decode_step", "rat_check_status",
           "rat_status_string", "rat_last_error", "rat_version", "rat_launch_count", "rat_debug_set_scan_stall",
           "rat_decode_step_noalloc", "rat_topk_stats_size", "rat_topk_build_stats", "rat_topk_decode_step",
           "rat_scan_prefill_paged", "rat_decode_step_paged"]


class RatError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s (%s)" % (msg, STATUS_NAMES.get(status, status)))
        self.status = status


STATUS_NAMES = {0: "RAT_OK", 1: "RAT_ERR_INVALID", 2: "RAT_ERR_UNSUPPORTED", 3: "RAT_ERR_CUDA",
                4: "RAT_ERR_TIMEOUT", 5: "RAT_ERR_WORKSPACE"}


class rat_cfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("dtype", ctypes.c_int), ("dil", ctypes.POINTER(ctypes.c_int32)),
                ("win", ctypes.POINTER(ctypes.c_int32)), ("recur", ctypes.POINTER(ctypes.c_uint8)),
                ("scale", ctypes.c_float), ("flags", ctypes.c_uint32), ("t0", ctypes.c_int), ("t_cap", ctypes.c_int)]


class rat_paged_cache(ctypes.Structure):
    _fields_ = [("pool_k", ctypes.c_void_p), ("pool_v", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
                ("page_rows", ctypes.c_int), ("pages_per_seq", ctypes.c_int), ("num_pages", ctypes.c_int)]


_lib = None


def load_library(path=LIB_PATH):
    """Load librat.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("librat.so not found at %s: run recurrence_augmented_dilated_gated_b200/build.py" % path)
    lib = ctypes.CDLL(path)
    P, S, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    cfgp = ctypes.POINTER(rat_cfg)
    lib.rat_workspace_size.argtypes = [cfgp, I, I]
    lib.rat_workspace_size.restype = S
    lib.rat_workspace_init.argtypes = [P, S, P]
    lib.rat_cache_rows.argtypes = [cfgp, I]
    lib.rat_cache_rows.restype = ctypes.c_int64
    lib.rat_scan_prefill.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, I, P, S, P]
    lib.rat_dilated_attn_prefill.argtypes = [cfgp, P, P, P, P, P, P, S, P]
    lib.rat_mix_prefill.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P]
    lib.rat_decode_step.argtypes = [cfgp, P, P, P, P, P, P, P, P, I, P, P, P, P, S, P]
    lib.rat_decode_step_noalloc.argtypes = [cfgp, P, P, P, P, P, P, P, P, I, P, P, P, P]
    lib.rat_topk_stats_size.argtypes = [cfgp, I, I]
    lib.rat_topk_stats_size.restype = S
    lib.rat_topk_build_stats.argtypes = [cfgp, I, I, P, I, P, P]
    lib.rat_topk_decode_step.argtypes = [cfgp, I, I, I, P, P, P, P, P, P, P, P, I, P, P, P, P, P, P, S, P]
    pcp = ctypes.POINTER(rat_paged_cache)
    lib.rat_scan_prefill_paged.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, pcp, I, P, S, P]
    lib.rat_decode_step_paged.argtypes = [cfgp, P, P, P, P, P, P, pcp, I, P, P, P, P, S, P]
    lib.rat_check_status.argtypes = [P, P]
    lib.rat_status_string.argtypes = [I]
    lib.rat_status_string.restype = ctypes.c_char_p
    lib.rat_last_error.argtypes = []
    lib.rat_last_error.restype = ctypes.c_char_p
    lib.rat_version.restype = I
    lib.rat_launch_count.restype = ctypes.c_longlong
    lib.rat_debug_set_scan_stall.argtypes = [P, S, ctypes.c_int64, ctypes.c_int64, P]
    for name in ("rat_workspace_init", "rat_scan_prefill", "rat_dilated_attn_prefill", "rat_mix_prefill",
                 "rat_decode_step", "rat_check_status", "rat_debug_set_scan_stall", "rat_decode_step_noalloc",
                 "rat_topk_build_stats", "rat_topk_decode_step", "rat_scan_prefill_paged",
                 "rat_decode_step_paged"):
        getattr(lib, name).restype = I
    _lib = lib
    return lib


class Config:
    """Owns a rat_cfg and the host arrays it points to."""

    def __init__(self, B, T, H, d, dtype, dil, win, recur=None, scale=0.0, flags=0, t0=0, t_cap=0):
        self.dil = np.ascontiguousarray(dil, dtype=np.int32)
        self.win = np.ascontiguousarray(win, dtype=np.int32)
        self.recur = None if recur is None else np.ascontiguousarray(recur, dtype=np.uint8)
        assert self.dil.shape == (H,) and self.win.shape == (H,)
        if isinstance(dtype, torch.dtype):
            dtype = {torch.float32: RAT_F32, torch.bfloat16: RAT_BF16}[dtype]
        self.c = rat_cfg(B, T, H, d, dtype,
                         self.dil.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                         self.win.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                         None if self.recur is None else self.recur.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                         float(scale), int(flags), int(t0), int(t_cap))

    @property
    def torch_dtype(self):
        return torch.float32 if self.c.dtype == RAT_F32 else torch.bfloat16

    def replace(self, **kw):
        args = dict(B=self.c.B, T=self.c.T, H=self.c.H, d=self.c.d, dtype=self.c.dtype, dil=self.dil,
                    win=self.win, recur=self.recur, scale=self.c.scale, flags=self.c.flags, t0=self.c.t0,
                    t_cap=self.c.t_cap)
        args.update(kw)
        return Config(**args)

    def ref(self):
        return ctypes.byref(self.c)

    @property
    def history_shape(self):
        """Shape of kt / vt: [B, t_cap or t0 + T, H, d] (the history in a chunked prefill)."""
        return (self.c.B, self.c.t_cap or self.c.t0 + self.c.T, self.c.H, self.c.d)

    def gate_shape(self, tok):
        """Shape of the gate tensor for token tensors of shape `tok` (a second,
        leading axis of 2 with separate key and value gates)."""
        return ((2,) + tuple(tok)) if self.c.flags & RAT_FLAG_SEPARATE_GATES else tuple(tok)


def _ptr(t, name, dtype=None, shape=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError("%s is required" % name)
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch tensor" % name)
    if t.numel() > 0 and t.device.type != "cuda":
        raise ValueError("%s must be a CUDA tensor (the library has no CPU path)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    return t.data_ptr() or None


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc, what):
    if rc != RAT_OK:
        raise RatError(rc, "%s: %s" % (what, load_library().rat_last_error().decode()))


def rat_version():
    return load_library().rat_version()


def rat_launch_count():
    return load_library().rat_launch_count()


def rat_workspace_size(cfg, op, cache_cap=0):
    n = load_library().rat_workspace_size(cfg.ref(), int(op), int(cache_cap))
    if n == 0:
        raise RatError(RAT_ERR_INVALID, "rat_workspace_size: invalid configuration")
    return n


def rat_workspace_init(ws, stream=None):
    _check(load_library().rat_workspace_init(_ptr(ws, "ws"), ws.numel(), _stream(stream)), "rat_workspace_init")


def workspace(cfg, op, cache_cap=0, device="cuda"):
    """A zero-filled workspace tensor (uint8) of rat_workspace_size bytes, 256-byte aligned."""
    n = rat_workspace_size(cfg, op, cache_cap)
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def rat_cache_rows(cfg, cap):
    r = load_library().rat_cache_rows(cfg.ref(), int(cap))
    if r == 0:
        raise RatError(RAT_ERR_INVALID, "rat_cache_rows: invalid configuration or capacity")
    return r


def rat_scan_prefill(cfg, k, v, g, init_k=None, init_v=None, kt=None, vt=None, final_k=None, final_v=None,
                     cache_k=None, cache_v=None, cache_cap=0, ws=None, stream=None):
    c = cfg.c
    tok = (c.B, c.T, c.H, c.d)
    st = (c.B, c.H, c.d)
    dt = cfg.torch_dtype
    args = [_ptr(k, "k", dt, tok), _ptr(v, "v", dt, tok), _ptr(g, "g", dt, cfg.gate_shape(tok)),
            _ptr(init_k, "init_k", torch.float32, st, True), _ptr(init_v, "init_v", torch.float32, st, True),
            _ptr(kt, "kt", dt, cfg.history_shape, True), _ptr(vt, "vt", dt, cfg.history_shape, True),
            _ptr(final_k, "final_k", torch.float32, st, True), _ptr(final_v, "final_v", torch.float32, st, True),
            _ptr(cache_k, "cache_k", dt, None, True), _ptr(cache_v, "cache_v", dt, None, True), int(cache_cap),
            _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream)]
    _check(load_library().rat_scan_prefill(cfg.ref(), *args), "rat_scan_prefill")


def rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse=None, ws=None, stream=None):
    c = cfg.c
    tok = (c.B, c.T, c.H, c.d)
    dt = cfg.torch_dtype
    args = [_ptr(q, "q", dt, tok), _ptr(kt, "kt", dt, cfg.history_shape), _ptr(vt, "vt", dt, cfg.history_shape),
            _ptr(o, "o", dt, tok),
            _ptr(lse, "lse", torch.float32, (c.B, c.H, c.T), True), _ptr(ws, "ws", torch.uint8), ws.numel(),
            _stream(stream)]
    _check(load_library().rat_dilated_attn_prefill(cfg.ref(), *args), "rat_dilated_attn_prefill")


def rat_mix_prefill(cfg, q, k, v, g, init_k=None, init_v=None, o=None, lse=None, kt=None, vt=None,
                    final_k=None, final_v=None, ws=None, stream=None):
    c = cfg.c
    tok = (c.B, c.T, c.H, c.d)
    st = (c.B, c.H, c.d)
    dt = cfg.torch_dtype
    args = [_ptr(q, "q", dt, tok), _ptr(k, "k", dt, tok), _ptr(v, "v", dt, tok), _ptr(g, "g", dt, cfg.gate_shape(tok)),
            _ptr(init_k, "init_k", torch.float32, st, True), _ptr(init_v, "init_v", torch.float32, st, True),
            _ptr(o, "o", dt, tok), _ptr(lse, "lse", torch.float32, (c.B, c.H, c.T), True),
            _ptr(kt, "kt", dt, cfg.history_shape, True), _ptr(vt, "vt", dt, cfg.history_shape, True),
            _ptr(final_k, "final_k", torch.float32, st, True), _ptr(final_v, "final_v", torch.float32, st, True),
            _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream)]
    _check(load_library().rat_mix_prefill(cfg.ref(), *args), "rat_mix_prefill")


def rat_decode_step(cfg, q, k, v, g, state_k, state_v, cache_k, cache_v, cache_cap, pos, o, lse=None, ws=None,
                    stream=None):
    c = cfg.c
    tok = (c.B, c.H, c.d)
    dt = cfg.torch_dtype
    R = rat_cache_rows(cfg, cache_cap)
    cshape = (c.B, c.H, R, c.d)
    args = [_ptr(q, "q", dt, tok), _ptr(k, "k", dt, tok), _ptr(v, "v", dt, tok), _ptr(g, "g", dt, cfg.gate_shape(tok)),
            _ptr(state_k, "state_k", torch.float32, tok), _ptr(state_v, "state_v", torch.float32, tok),
            _ptr(cache_k, "cache_k", dt, cshape), _ptr(cache_v, "cache_v", dt, cshape), int(cache_cap),
            _ptr(pos, "pos", torch.int32, (c.B,)), _ptr(o, "o", dt, tok),
            _ptr(lse, "lse", torch.float32, (c.B, c.H), True), _ptr(ws, "ws", torch.uint8), ws.numel(),
            _stream(stream)]
    _check(load_library().rat_decode_step(cfg.ref(), *args), "rat_decode_step")


def rat_decode_step_noalloc(cfg, q, k, v, g, state_k, state_v, cache_k, cache_v, cache_cap, pos, o, lse=None,
                            stream=None):
    """rat_decode_step without a workspace: for callers that cannot allocate
    device memory while decoding (its scratch is a static 16 MiB array inside
    the library).  Calls whose kernels overlap on the GPU race on that array."""
    c = cfg.c
    tok = (c.B, c.H, c.d)
    dt = cfg.torch_dtype
    R = rat_cache_rows(cfg, cache_cap)
    cshape = (c.B, c.H, R, c.d)
    args = [_ptr(q, "q", dt, tok), _ptr(k, "k", dt, tok), _ptr(v, "v", dt, tok), _ptr(g, "g", dt, cfg.gate_shape(tok)),
            _ptr(state_k, "state_k", torch.float32, tok), _ptr(state_v, "state_v", torch.float32, tok),
            _ptr(cache_k, "cache_k", dt, cshape), _ptr(cache_v, "cache_v", dt, cshape), int(cache_cap),
            _ptr(pos, "pos", torch.int32, (c.B,)), _ptr(o, "o", dt, tok),
            _ptr(lse, "lse", torch.float32, (c.B, c.H), True), _stream(stream)]
    _check(load_library().rat_decode_step_noalloc(cfg.ref(), *args), "rat_decode_step_noalloc")


def rat_topk_stats_size(cfg, block, cache_cap):
    n = load_library().rat_topk_stats_size(cfg.ref(), int(block), int(cache_cap))
    if n == 0:
        raise RatError(RAT_ERR_INVALID, "rat_topk_stats_size: " + load_library().rat_last_error().decode())
    return n


def topk_stats_shape(cfg, block, cache_cap):
    """Shape of the fp32 block-statistics tensor: [B, H, ceil(cap / block), 2, d]."""
    c = cfg.c
    return (c.B, c.H, -(-int(cache_cap) // int(block)), 2, c.d)


def rat_topk_build_stats(cfg, block, mode, cache_k, cache_cap, stats, stream=None):
    c = cfg.c
    R = rat_cache_rows(cfg, cache_cap)
    args = [int(block), int(mode), _ptr(cache_k, "cache_k", cfg.torch_dtype, (c.B, c.H, R, c.d)), int(cache_cap),
            _ptr(stats, "stats", torch.float32, topk_stats_shape(cfg, block, cache_cap)), _stream(stream)]
    _check(load_library().rat_topk_build_stats(cfg.ref(), *args), "rat_topk_build_stats")


def rat_topk_decode_step(cfg, block, topk, mode, q, k, v, g, state_k, state_v, cache_k, cache_v, cache_cap, stats,
                         pos, o, lse=None, sel=None, ws=None, stream=None):
    c = cfg.c
    tok = (c.B, c.H, c.d)
    dt = cfg.torch_dtype
    R = rat_cache_rows(cfg, cache_cap)
    cshape = (c.B, c.H, R, c.d)
    args = [int(block), int(topk), int(mode),
            _ptr(q, "q", dt, tok), _ptr(k, "k", dt, tok), _ptr(v, "v", dt, tok), _ptr(g, "g", dt, cfg.gate_shape(tok)),
            _ptr(state_k, "state_k", torch.float32, tok), _ptr(state_v, "state_v", torch.float32, tok),
            _ptr(cache_k, "cache_k", dt, cshape), _ptr(cache_v, "cache_v", dt, cshape), int(cache_cap),
            _ptr(stats, "stats", torch.float32, topk_stats_shape(cfg, block, cache_cap)),
            _ptr(pos, "pos", torch.int32, (c.B,)), _ptr(o, "o", dt, tok),
            _ptr(lse, "lse", torch.float32, (c.B, c.H), True),
            _ptr(sel, "sel", torch.int32, (c.B, c.H, int(topk)), True),
            _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream)]
    _check(load_library().rat_topk_decode_step(cfg.ref(), *args), "rat_topk_decode_step")


def paged_cache(cfg, pool_k, pool_v, page_table, cache_cap):
    """A rat_paged_cache over torch tensors: pools [num_pages, H, page_rows, d]
    in the cfg's dtype and a device int32 table [B, pages_per_seq]."""
    c = cfg.c
    if pool_k.dim() != 4 or pool_k.shape[1] != c.H or pool_k.shape[3] != c.d:
        raise ValueError("pool_k must be [num_pages, H, page_rows, d]")
    n, _, P, _ = pool_k.shape
    _ptr(pool_k, "pool_k", cfg.torch_dtype)
    _ptr(pool_v, "pool_v", cfg.torch_dtype, tuple(pool_k.shape))
    _ptr(page_table, "page_table", torch.int32)
    if page_table.dim() != 2 or page_table.shape[0] != c.B:
        raise ValueError("page_table must be [B, pages_per_seq]")
    return rat_paged_cache(pool_k.data_ptr(), pool_v.data_ptr(), page_table.data_ptr(), int(P),
                           int(page_table.shape[1]), int(n))


def rat_scan_prefill_paged(cfg, k, v, g, init_k=None, init_v=None, kt=None, vt=None, final_k=None, final_v=None,
                           cache=None, cache_cap=0, ws=None, stream=None):
    """rat_scan_prefill into a paged cache (a rat_paged_cache from paged_cache())."""
    c = cfg.c
    tok = (c.B, c.T, c.H, c.d)
    st = (c.B, c.H, c.d)
    dt = cfg.torch_dtype
    args = [_ptr(k, "k", dt, tok), _ptr(v, "v", dt, tok), _ptr(g, "g", dt, cfg.gate_shape(tok)),
            _ptr(init_k, "init_k", torch.float32, st, True), _ptr(init_v, "init_v", torch.float32, st, True),
            _ptr(kt, "kt", dt, cfg.history_shape, True), _ptr(vt, "vt", dt, cfg.history_shape, True),
            _ptr(final_k, "final_k", torch.float32, st, True), _ptr(final_v, "final_v", torch.float32, st, True),
            ctypes.byref(cache), int(cache_cap), _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream)]
    _check(load_library().rat_scan_prefill_paged(cfg.ref(), *args), "rat_scan_prefill_paged")


def rat_decode_step_paged(cfg, q, k, v, g, state_k, state_v, cache, cache_cap, pos, o, lse=None, ws=None,
                          stream=None):
    """rat_decode_step over a paged cache (a rat_paged_cache from paged_cache())."""
    c = cfg.c
    tok = (c.B, c.H, c.d)
    dt = cfg.torch_dtype
    args = [_ptr(q, "q", dt, tok), _ptr(k, "k", dt, tok), _ptr(v, "v", dt, tok), _ptr(g, "g", dt, cfg.gate_shape(tok)),
            _ptr(state_k, "state_k", torch.float32, tok), _ptr(state_v, "state_v", torch.float32, tok),
            ctypes.byref(cache), int(cache_cap), _ptr(pos, "pos", torch.int32, (c.B,)), _ptr(o, "o", dt, tok),
            _ptr(lse, "lse", torch.float32, (c.B, c.H), True), _ptr(ws, "ws", torch.uint8), ws.numel(),
            _stream(stream)]
    _check(load_library().rat_decode_step_paged(cfg.ref(), *args), "rat_decode_step_paged")


def rat_check_status(ws, stream=None):
    """Synchronise and raise RatError if the kernels recorded a device-side error."""
    _check(load_library().rat_check_status(_ptr(ws, "ws"), _stream(stream)), "rat_check_status")


def rat_debug_set_scan_stall(ws, ticket, spin_limit_ns=0, stream=None):
    _check(load_library().rat_debug_set_scan_stall(_ptr(ws, "ws"), ws.numel(), int(ticket), int(spin_limit_ns),
                                                   _stream(stream)), "rat_debug_set_scan_stall")


# ----------------------------------------------------------------- conveniences


def mix_prefill(cfg, q, k, v, g, init_k=None, init_v=None, want_kv=False, want_lse=True, ws=None, stream=None):
    """Allocate outputs with torch and run rat_mix_prefill.  Returns a dict.
    (A chunked prefill, t0 > 0, calls rat_mix_prefill with its kt/vt history.)"""
    c = cfg.c
    if c.t0 > 0:
        raise ValueError("mix_prefill allocates its own kt/vt: with t0 > 0 call rat_mix_prefill with the history")
    dev = q.device
    o = torch.empty_like(q)
    lse = torch.empty((c.B, c.H, c.T), dtype=torch.float32, device=dev) if want_lse else None
    kt = torch.empty_like(k) if want_kv else None
    vt = torch.empty_like(v) if want_kv else None
    fk = torch.empty((c.B, c.H, c.d), dtype=torch.float32, device=dev)
    fv = torch.empty_like(fk)
    if ws is None:
        ws = workspace(cfg, RAT_OP_MIX_CALLER_KV if want_kv else RAT_OP_MIX, device=dev)
    rat_mix_prefill(cfg, q, k, v, g, init_k, init_v, o, lse, kt, vt, fk, fv, ws, stream)
    return dict(o=o, lse=lse, kt=kt, vt=vt, final_k=fk, final_v=fv, ws=ws)

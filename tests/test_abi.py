"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

* librat.so builds, loads and exports every function include/rat.h declares;
* argument validation returns the documented status before any launch;
* workspace sizes and the decode-cache layout are as documented.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import recurrence_augmented_dilated_gated_b200 as rat
from recurrence_augmented_dilated_gated_b200 import build as rat_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    rat_build.build()
    return rat.load_library()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "rat.h")).read()
    return sorted(set(re.findall(r"RAT_API\s+[\w\s\*]+?\b(rat_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(rat.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.rat_version() == 101


def test_status_strings(lib):
    for s in range(6):
        assert lib.rat_status_string(s).decode().startswith(rat.STATUS_NAMES[s])


def cfg(**kw):
    a = dict(B=1, T=100, H=2, d=128, dtype=rat.RAT_BF16, dil=[4, 4], win=[0, 8], recur=None, scale=0.0)
    a.update(kw)
    return rat.Config(**a)


def test_workspace_size_rejects_bad_configs(lib):
    c = cfg()
    assert lib.rat_workspace_size(c.ref(), rat.RAT_OP_MIX, 0) > 0
    for bad in (cfg(d=96), cfg(d=32), cfg(H=300, dil=[1] * 300, win=[0] * 300), cfg(dil=[0, 4]),
                cfg(win=[-1, 0]), cfg(dtype=7), cfg(B=-1)):
        assert lib.rat_workspace_size(bad.ref(), rat.RAT_OP_MIX, 0) == 0
    assert lib.rat_workspace_size(c.ref(), 99, 0) == 0
    assert lib.rat_workspace_size(c.ref(), rat.RAT_OP_DECODE, 0) == 0  # decode needs a capacity


def test_workspace_grows_with_what_it_holds(lib):
    c = cfg(T=4096)
    scan = lib.rat_workspace_size(c.ref(), rat.RAT_OP_SCAN, 0)
    mix = lib.rat_workspace_size(c.ref(), rat.RAT_OP_MIX, 0)
    mixkv = lib.rat_workspace_size(c.ref(), rat.RAT_OP_MIX_CALLER_KV, 0)
    kv_bytes = 2 * 1 * 4096 * 2 * 128 * 2
    assert mix - mixkv >= kv_bytes and mixkv > scan
    d1 = lib.rat_workspace_size(c.ref(), rat.RAT_OP_DECODE, 1000)
    d2 = lib.rat_workspace_size(c.ref(), rat.RAT_OP_DECODE, 100000)
    assert d2 > d1 > 0


def test_decode_split_adapts_to_the_batch(lib):
    # Decode splits each (b, h) slab into work items of at most 2048 rows, and
    # halves that (down to 256) while batch x items would leave SMs idle.  The
    # workspace holds one (d + 2)-float partial per item, so its size per batch
    # entry shows the split: 16 heads at D = 16, capacity 32768 (2048-row slabs).
    def part_floats_per_b(B):
        c = cfg(B=B, H=16, dil=[16] * 16, win=[0] * 16)
        return lib.rat_workspace_size(c.ref(), rat.RAT_OP_DECODE, 32768)
    big, small = part_floats_per_b(256), part_floats_per_b(1)
    items_big = 16 * 1      # one 2048-row item per head already fills the GPU at batch 256
    items_small = 16 * 8    # batch 1: 256-row items
    per_item = (128 + 2) * 4
    assert big >= 256 * items_big * per_item
    assert big < 256 * 2 * items_big * per_item      # not split further
    assert small >= items_small * per_item            # split down to 256-row items


def test_cache_rows_layout(lib):
    # rows per (b,h) block = max_h D_h * ceil(cap / D_h)
    c = cfg(H=3, dil=[1, 16, 64], win=[0, 0, 256])
    for cap in (1, 63, 64, 65, 4096, 33792):
        expect = max(D * -(-cap // D) for D in (1, 16, 64))
        assert lib.rat_cache_rows(c.ref(), cap) == expect
    assert lib.rat_cache_rows(c.ref(), 0) == 0



def test_cache_rows_layout_fixed_grid(lib):
    # fixed grid: ceil(cap / D) grid rows, plus a ring of W rows when D > 1 and W > 0
    c = cfg(H=4, dil=[1, 16, 64, 8], win=[32, 0, 256, 0], flags=rat.RAT_FLAG_GRID_DILATION)
    for cap in (1, 63, 64, 65, 4096, 33792):
        expect = max(-(-cap // D) + (W if D > 1 else 0) for D, W in ((1, 32), (16, 0), (64, 256), (8, 0)))
        assert lib.rat_cache_rows(c.ref(), cap) == expect
    # the decode plan strides the cache by the same row count (workspace stays defined)
    assert lib.rat_workspace_size(c.ref(), rat.RAT_OP_DECODE, 4096) > 0


def test_unknown_flags_are_rejected(lib):
    assert lib.rat_workspace_size(cfg(flags=8).ref(), rat.RAT_OP_MIX, 0) == 0
    for f in (rat.RAT_FLAG_GRID_DILATION, rat.RAT_FLAG_DEDUPE, rat.RAT_FLAG_SEPARATE_GATES,
              rat.RAT_FLAG_GRID_DILATION | rat.RAT_FLAG_DEDUPE | rat.RAT_FLAG_SEPARATE_GATES):
        assert lib.rat_workspace_size(cfg(flags=f).ref(), rat.RAT_OP_MIX, 0) > 0



def test_topk_sizes_and_argument_checks(lib):
    c = cfg(B=2, H=2, dil=[1, 1], win=[0, 0])
    # statistics: [B, H, ceil(cap / block), 2, d] fp32
    assert lib.rat_topk_stats_size(c.ref(), 64, 4000) == 2 * 2 * 63 * 2 * 128 * 4
    assert lib.rat_topk_stats_size(cfg().ref(), 64, 4096) == 0          # dilated heads: not the dense layout
    assert lib.rat_topk_stats_size(cfg(dil=[1, 1]).ref(), 64, 4096) == 0  # a window
    assert lib.rat_topk_stats_size(c.ref(), 0, 4096) == 0
    assert lib.rat_topk_stats_size(c.ref(), 1, 16385) == 0               # more blocks than the kernel holds
    assert lib.rat_workspace_size(c.ref(), rat.RAT_OP_TOPK_DECODE, 4096) == 256
    P = 16
    for block, topk, mode in ((64, 65, 0), (64, -1, 0), (64, 4, 2), (0, 4, 0)):
        rc = lib.rat_topk_decode_step(c.ref(), block, topk, mode, P, P, P, P, P, P, P, P, 4096, P, P, P, None,
                                      None, 256, 256, None)
        assert rc == rat.RAT_ERR_INVALID, (block, topk, mode)
    rc = lib.rat_topk_build_stats(c.replace(T=5000).ref(), 64, 0, P, 4096, P, None)
    assert rc == rat.RAT_ERR_INVALID     # more tokens than the cache holds
    # the step streams cache rows and block statistics through shared memory in
    # 16-byte copies: a cache or statistics pointer off that alignment is
    # refused before anything is launched (the other arguments are valid)
    good = dict(q=P, k=P, v=P, g=P, sk=P, sv=P, ck=P, cv=P, stats=P, pos=P, o=P)
    for name in ("ck", "cv", "stats"):
        a = dict(good)
        a[name] = P + 4
        rc = lib.rat_topk_decode_step(c.ref(), 64, 4, 0, a["q"], a["k"], a["v"], a["g"], a["sk"], a["sv"], a["ck"],
                                      a["cv"], 4096, a["stats"], a["pos"], a["o"], None, None, 256, 256, None)
        assert rc == rat.RAT_ERR_INVALID, name
        assert b"16-byte aligned" in lib.rat_last_error(), name



def test_paged_cache_descriptor_checks(lib):
    # host-side checks of the page descriptor, before any launch
    c = cfg(B=2, H=2, dil=[1, 4], win=[0, 8])
    cap = 1000
    R = lib.rat_cache_rows(c.ref(), cap)
    P = 16

    def step(desc):
        return lib.rat_decode_step_paged(c.ref(), P, P, P, P, P, P, ctypes.byref(desc), cap, P, P, None, 256, 1 << 30,
                                         None)

    good = dict(pool_k=16, pool_v=32, page_table=48, page_rows=64, pages_per_seq=-(-R // 64), num_pages=64)
    for bad in (dict(page_rows=0), dict(num_pages=0), dict(pages_per_seq=-(-R // 64) - 1), dict(pool_k=None),
                dict(page_table=8)):
        d = dict(good)
        d.update(bad)
        assert step(rat.rat_paged_cache(**d)) == rat.RAT_ERR_INVALID, bad
    assert lib.rat_decode_step_paged(c.ref(), P, P, P, P, P, P, None, cap, P, P, None, 256, 1 << 30,
                                     None) == rat.RAT_ERR_INVALID



def test_chunked_prefill_arguments(lib):
    # t_cap must hold the history; a chunk after the first needs the caller's kt/vt
    assert lib.rat_workspace_size(cfg(t0=100, t_cap=150).ref(), rat.RAT_OP_SCAN, 0) == 0     # T = 100
    assert lib.rat_workspace_size(cfg(t0=100, t_cap=200).ref(), rat.RAT_OP_SCAN, 0) > 0
    assert lib.rat_workspace_size(cfg(t0=-1).ref(), rat.RAT_OP_SCAN, 0) == 0
    c = cfg(t0=100)
    P = 16
    rc = lib.rat_mix_prefill(c.ref(), P, P, P, P, None, None, P, None, None, None, None, None, 256, 1 << 40, None)
    assert rc == rat.RAT_ERR_INVALID


def call_scan(lib, c, **ptrs):
    P = dict(k=16, v=16, g=16, init_k=None, init_v=None, kt=16, vt=16, fk=None, fv=None, ck=None, cv=None, cap=0,
             ws=256, wsb=1 << 40)
    P.update(ptrs)
    return lib.rat_scan_prefill(c.ref(), P["k"], P["v"], P["g"], P["init_k"], P["init_v"], P["kt"], P["vt"],
                                P["fk"], P["fv"], P["ck"], P["cv"], P["cap"], P["ws"], P["wsb"], None)


def test_argument_errors_return_before_launch(lib):
    # fake (never dereferenced) addresses: every call below must fail in validation
    c = cfg()
    assert call_scan(lib, c, k=None) == rat.RAT_ERR_INVALID
    assert call_scan(lib, c, k=8) == rat.RAT_ERR_INVALID                     # misaligned
    assert call_scan(lib, c, kt=None, vt=None) == rat.RAT_ERR_INVALID         # no output
    assert call_scan(lib, c, vt=None) == rat.RAT_ERR_INVALID                  # unpaired
    assert call_scan(lib, c, ck=16, cv=16, cap=50) == rat.RAT_ERR_INVALID    # cap < T
    assert call_scan(lib, c, wsb=16) == rat.RAT_ERR_WORKSPACE
    assert call_scan(lib, c, ws=None) == rat.RAT_ERR_INVALID
    assert call_scan(lib, c, ws=272) == rat.RAT_ERR_INVALID                   # ws not 256-aligned
    assert call_scan(lib, cfg(d=96)) == rat.RAT_ERR_UNSUPPORTED
    assert b"aligned" in lib.rat_last_error() or len(lib.rat_last_error()) > 0
    bad = lib.rat_dilated_attn_prefill(c.ref(), 16, 16, 16, None, None, 256, 1 << 40, None)
    assert bad == rat.RAT_ERR_INVALID
    bad = lib.rat_decode_step(c.ref(), 16, 16, 16, 16, 16, 16, 16, 16, 0, 16, 16, None, 256, 1 << 40, None)
    assert bad == rat.RAT_ERR_INVALID                                          # cap < 1
    assert lib.rat_check_status(None, None) == rat.RAT_ERR_INVALID


def test_binding_refuses_cpu_tensors():
    c = cfg(T=8)
    x = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        rat.rat_scan_prefill(c, x, x, x, kt=x, vt=x, ws=torch.zeros(1 << 20, dtype=torch.uint8))

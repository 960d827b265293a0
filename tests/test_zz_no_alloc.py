"""rat_decode_step_noalloc: the decode step for callers that cannot allocate
device memory while they decode (an engine plugin given no scratch buffer, a
serving loop with a fixed memory budget).  Its scratch is a static 16 MiB array
inside the library instead of a caller workspace.

The two entry points run the same step plan and the same kernel on the same
inputs, so their results must be bit-identical: the GPU tests run decode steps
in a row through the C ABI with both, on separate copies of the cache and
state, and compare outputs, lse, both states and both caches with exact
equality (any wrong offset into the static scratch would show).  One case runs
at the largest batch whose step still fits the scratch.  The CPU tests check
that both entry points refuse the same bad arguments with the same status.
The file is named so that pytest collects it last.
"""
import pytest
import torch

import workloads as wl

rat = pytest.importorskip("recurrence_augmented_dilated_gated_b200")

SCRATCH_BYTES = 16 << 20


def test_noalloc_rejects_steps_beyond_its_scratch():
    # 4096 * 16 heads * (1 split + tail) * 130 floats > 16 MiB: refused before any launch
    cfg = rat.Config(4096, 1, 16, 128, rat.RAT_BF16, [16] * 16, [0] * 16)
    lib = rat.load_library()
    rc = lib.rat_decode_step_noalloc(cfg.ref(), *([16] * 8), 4096, 16, 16, None, None)
    assert rc == rat.RAT_ERR_UNSUPPORTED
    assert b"16 MiB" in lib.rat_last_error()


def test_noalloc_and_workspace_decode_refuse_alike():
    # the same argument checker serves both: every bad call returns the same
    # status from each (no pointer is dereferenced; nothing is launched)
    lib = rat.load_library()
    ok = 1 << 20   # a fake, 16-byte aligned address
    good = dict(cfg=rat.Config(2, 1, 2, 128, rat.RAT_BF16, [4, 4], [0, 8]), ptrs=[ok] * 8, cap=64, pos=ok, o=ok,
                lse=None)
    cases = [
        dict(cfg=rat.Config(2, 1, 2, 96, rat.RAT_BF16, [4, 4], [0, 0])),               # d unsupported
        dict(cfg=rat.Config(2, 1, 300, 128, rat.RAT_BF16, [1] * 300, [0] * 300)),       # H > 256
        dict(cfg=rat.Config(2, 1, 2, 128, 7, [4, 4], [0, 0])),                          # dtype
        dict(cfg=rat.Config(2, 1, 2, 128, rat.RAT_BF16, [0, 4], [0, 0])),               # dil < 1
        dict(cfg=rat.Config(2, 1, 2, 128, rat.RAT_BF16, [4, 4], [-1, 0])),              # win < 0
        dict(cfg=rat.Config(2, 1, 2, 128, rat.RAT_BF16, [4, 4], [0, 0], flags=64)),     # unknown flag
        dict(ptrs=[0] + [ok] * 7),                                                      # q NULL
        dict(ptrs=[ok] * 3 + [ok + 8] + [ok] * 4),                                      # g misaligned
        dict(pos=0),                                                                    # pos NULL
        dict(o=ok + 4),                                                                 # o misaligned
        dict(lse=ok + 4),                                                               # lse misaligned
        dict(cap=0),                                                                    # cache_cap < 1
    ]
    # every case breaks one argument of a valid call, so each fails its checks
    # before the workspace (a fake address here) is looked at
    for i, case in enumerate(cases):
        a = dict(good)
        a.update(case)
        p = a["ptrs"]
        rc_ws = lib.rat_decode_step(a["cfg"].ref(), *p, a["cap"], a["pos"], a["o"], a["lse"], ok, 1 << 30, None)
        err_ws = lib.rat_last_error()
        rc_na = lib.rat_decode_step_noalloc(a["cfg"].ref(), *p, a["cap"], a["pos"], a["o"], a["lse"], None)
        err_na = lib.rat_last_error()
        assert rc_ws != rat.RAT_OK, i
        assert rc_na == rc_ws, (i, rc_na, rc_ws, err_na, err_ws)
        assert err_na == err_ws, (i, err_na, err_ws)


def run_both(B, T, H, d, dil, win, recur, steps, seed):
    """Prefill T tokens, then `steps` decode steps through each entry point on
    its own copy of the cache and state; assert bit-identical results."""
    dev = "cuda"
    dtype = torch.bfloat16
    cap = T + steps
    q, k, v, g = (x.to(dev) for x in wl.prefill_inputs(B, cap, H, d, 2.0, dtype, seed=seed))
    cfg = rat.Config(B, T, H, d, dtype, dil, win, recur)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=dev)
    cv = torch.zeros_like(ck)
    sk = torch.empty(B, H, d, device=dev)
    sv = torch.empty_like(sk)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_scan_prefill(cfg, k[:, :T].contiguous(), v[:, :T].contiguous(), g[:, :T].contiguous(), None, None,
                         None, None, sk, sv, ck, cv, cap, ws)
    rat.rat_check_status(ws)
    # two independent copies of the decode state: one per entry point
    a = dict(ck=ck.clone(), cv=cv.clone(), sk=sk.clone(), sv=sv.clone())
    b = dict(ck=ck, cv=cv, sk=sk, sv=sv)
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    for s in range(steps):
        t = T + s
        pos = torch.full((B,), t, dtype=torch.int32, device=dev)
        tok = [x[:, t].contiguous() for x in (q, k, v, g)]
        oa, la = torch.empty(B, H, d, dtype=dtype, device=dev), torch.empty(B, H, device=dev)
        ob, lb = torch.full_like(oa, float("nan")), torch.full_like(la, float("nan"))
        rat.rat_decode_step(cfg, *tok, a["sk"], a["sv"], a["ck"], a["cv"], cap, pos, oa, la, wsd)
        rat.rat_decode_step_noalloc(cfg, *tok, b["sk"], b["sv"], b["ck"], b["cv"], cap, pos, ob, lb)
        torch.cuda.synchronize()
        assert torch.equal(ob, oa), "o differs at step %d" % s
        assert torch.equal(lb, la), "lse differs at step %d" % s
        for key in ("sk", "sv", "ck", "cv"):
            assert torch.equal(b[key], a[key]), "%s differs after step %d" % (key, s)
    rat.rat_check_status(wsd)


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode():
    # a hybrid of heads: dense without recurrence, windowed, long residue slab
    run_both(B=4, T=700, H=3, d=128, dil=[1, 4, 16], win=[0, 32, 0], recur=[0, 1, 1], steps=2, seed=77)


@pytest.mark.gpu
def test_noalloc_decode_at_the_largest_batch_its_scratch_holds():
    # the largest batch whose step fits the 16 MiB scratch (the workspace the
    # other entry point needs is header + the same scratch), two steps in a row
    H, d, T, steps = 16, 128, 100, 2
    dil, win = [16] * H, [0] * H
    size = lambda B: rat.rat_workspace_size(rat.Config(B, T, H, d, torch.bfloat16, dil, win), rat.RAT_OP_DECODE,
                                            T + steps)
    lo, hi = 1, 1 << 16
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if size(mid) <= SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid - 1
    B = lo
    assert size(B) <= SCRATCH_BYTES < size(B + 1)
    run_both(B=B, T=T, H=H, d=d, dil=dil, win=win, recur=None, steps=steps, seed=78)

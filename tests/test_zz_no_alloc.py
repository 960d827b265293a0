"""rat_decode_step_noalloc: the decode step for callers that cannot allocate
device memory while they decode (an engine plugin given no scratch buffer, a
serving loop with a fixed memory budget).  Its scratch is a static 16 MiB array
inside the library instead of a caller workspace.

The GPU test runs two decode steps in a row through the C ABI with both entry
points, on separate copies of the cache and state, and checks that the
workspace-free call gives the same outputs, states and cache rows as
rat_decode_step, within the tolerance the parity tests use (relative L2 1e-2
for bf16).  The file is named so that pytest collects it last.
"""
import pytest
import torch

import workloads as wl
from parity import assert_close

rat = pytest.importorskip("recurrence_augmented_dilated_gated_b200")


def test_noalloc_rejects_steps_beyond_its_scratch():
    # 4096 * 16 heads * (1 split + tail) * 130 floats > 16 MiB: refused before any launch
    cfg = rat.Config(4096, 1, 16, 128, rat.RAT_BF16, [16] * 16, [0] * 16)
    lib = rat.load_library()
    rc = lib.rat_decode_step_noalloc(cfg.ref(), *([16] * 8), 4096, 16, 16, None, None)
    assert rc == rat.RAT_ERR_UNSUPPORTED
    assert b"16 MiB" in lib.rat_last_error()


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode():
    dev = "cuda"
    B, T, H, d = 4, 700, 3, 128
    dil, win, recur = [1, 4, 16], [0, 32, 0], [0, 1, 1]
    dtype = torch.bfloat16
    steps = 2
    cap = T + steps
    q, k, v, g = (x.to(dev) for x in wl.prefill_inputs(B, cap, H, d, 2.0, dtype, seed=77))
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
    b = dict(ck=ck.clone(), cv=cv.clone(), sk=sk.clone(), sv=sv.clone())
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    for s in range(steps):
        t = T + s
        pos = torch.full((B,), t, dtype=torch.int32, device=dev)
        tok = [x[:, t].contiguous() for x in (q, k, v, g)]
        oa, la = torch.empty(B, H, d, dtype=dtype, device=dev), torch.empty(B, H, device=dev)
        ob, lb = torch.empty_like(oa), torch.empty_like(la)
        rat.rat_decode_step(cfg, *tok, a["sk"], a["sv"], a["ck"], a["cv"], cap, pos, oa, la, wsd)
        rat.rat_decode_step_noalloc(cfg, *tok, b["sk"], b["sv"], b["ck"], b["cv"], cap, pos, ob, lb)
        torch.cuda.synchronize()
        assert_close(ob, oa.float().cpu().numpy(), dtype, "o step %d" % s)
        assert_close(lb, la.float().cpu().numpy(), dtype, "lse step %d" % s)
    rat.rat_check_status(wsd)
    for key in ("sk", "sv", "ck", "cv"):
        assert_close(b[key], a[key].float().cpu().numpy(), dtype, key)

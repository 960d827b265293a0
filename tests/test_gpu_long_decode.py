"""GPU parity of the decode workloads over their whole horizon.

The decode benchmark runs batch 256 (16 heads of 128, D = 16) for 1024 steps
after a prefilled context of 4096, 16384 or 32768 tokens, and the hybrid
workload's batch 128 (32 heads: 4 dense, 28 with D = 64 and W = 256) for 256
steps after 65536 tokens ("RAT+: Train Dense, Infer Sparse", Figure 2: decode
at batch 256 and 128).  These tests run exactly those steps on the GPU, at the
full batch and head count, and compare sampled batch entries and heads with the
fp64 oracle at EVERY step, plus the recurrent state after the last one:

  * the cache is filled the way the benchmark fills it: rat_scan_prefill over
    batch chunks whose k, v, g come from their own seeds, writing straight into
    the cache and the running state;
  * step s feeds the tokens of workloads.token_inputs(seed = 5000 + s) at
    position ctx + s for every entry;
  * the oracle scans the sampled entries' whole sequences (prefill tokens,
    then the decoded ones) and computes each decoded row from the definition.

Unused cache rows start as NaN, so a step that read a row it should not would
turn its output non-finite.  The bar is the operator's (relative L2 1e-2 for
bf16), per step; the worst single (entry, head) row of any step must also stay
within 5e-2, so one bad split item cannot hide in the pooled norm.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import assert_close, f64

rat = pytest.importorskip("recurrence_augmented_dilated_gated_b200")

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DEV = "cuda"


def long_decode_check(w, ctx, steps, check_b, check_h, fill_chunk, seed=0):
    dtype = torch.bfloat16
    B, H, d = w.decode_batch, w.H, w.d
    torch.cuda.empty_cache()
    cap = ctx + steps
    cfg = rat.Config(B, ctx, H, d, dtype, w.dil, w.win, w.recur)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.full((B, H, R, d), float("nan"), dtype=dtype, device=DEV)
    cv = torch.full_like(ck, float("nan"))
    sk = torch.empty(B, H, d, device=DEV)
    sv = torch.empty_like(sk)
    per_b = H * R * d
    hsel = torch.tensor(check_h, device=DEV)

    # prefill of the cache, batch chunk by batch chunk (inputs per chunk seed)
    ccfg = rat.Config(fill_chunk, ctx, H, d, dtype, w.dil, w.win, w.recur)
    wsc = rat.workspace(ccfg, rat.RAT_OP_SCAN)
    hist = {}  # sampled entry -> host (k, v, g) [ctx, len(check_h), d]
    for c, b0 in enumerate(range(0, B, fill_chunk)):
        _, k, v, g = wl.prefill_inputs(fill_chunk, ctx, H, d, w.gate_mean, dtype, device=DEV, seed=seed + 1 + c)
        rat.rat_scan_prefill(ccfg, k, v, g, None, None, None, None, sk[b0:b0 + fill_chunk], sv[b0:b0 + fill_chunk],
                             ck.view(-1)[b0 * per_b:(b0 + fill_chunk) * per_b],
                             cv.view(-1)[b0 * per_b:(b0 + fill_chunk) * per_b], cap, ws=wsc)
        for b in check_b:
            if b0 <= b < b0 + fill_chunk:
                hist[b] = tuple(f64(x[b - b0][:, hsel]) for x in (k, v, g))
        del k, v, g
    rat.rat_check_status(wsc)
    del wsc

    # the decode steps; the sampled units' inputs and outputs are kept
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    bsel = torch.tensor(check_b, device=DEV)
    pick = lambda x: x[bsel][:, hsel]
    o = torch.empty(B, H, d, dtype=dtype, device=DEV)
    lse = torch.empty(B, H, device=DEV)
    tok_in, got_o, got_l = [], [], []
    for s in range(steps):
        q1, k1, v1, g1 = wl.token_inputs(B, H, d, w.gate_mean, dtype, device=DEV, seed=5000 + s)
        pos = torch.full((B,), ctx + s, dtype=torch.int32, device=DEV)
        rat.rat_decode_step(cfg, q1, k1, v1, g1, sk, sv, ck, cv, cap, pos, o, lse, wsd)
        tok_in.append(torch.stack([pick(x) for x in (q1, k1, v1, g1)]))
        got_o.append(pick(o))
        got_l.append(pick(lse))
    rat.rat_check_status(wsd)
    tok = f64(torch.stack(tok_in))          # [steps, 4, nb, nh, d]
    got_o = f64(torch.stack(got_o))         # [steps, nb, nh, d]
    got_l = f64(torch.stack(got_l))         # [steps, nb, nh]
    got_sk, got_sv = pick(sk), pick(sv)
    del ck, cv, wsd
    torch.cuda.empty_cache()

    # the oracle over the sampled units' whole sequences
    nb, nh = len(check_b), len(check_h)
    Tt = ctx + steps
    seq = np.zeros((4, nb, Tt, nh, d))
    for i, b in enumerate(check_b):
        for j in range(3):                  # k, v, g of the prefill; q is unused there
            seq[1 + j, i, :ctx] = hist[b][j]
    seq[:, :, ctx:] = tok.transpose(1, 2, 0, 3, 4)
    recur = [w.recur[h] for h in check_h]
    dil = [w.dil[h] for h in check_h]
    win = [w.win[h] for h in check_h]
    kt, fk = oracle.scan(seq[1], seq[3], None, recur)
    vt, fv = oracle.scan(seq[2], seq[3], None, recur)
    rows = np.array([(i, j, ctx + s) for s in range(steps) for i in range(nb) for j in range(nh)])
    ro, rl = oracle.attn_rows(seq[0], kt, vt, dil, win, rows, parts=3)
    ro = ro.reshape(steps, nb, nh, d)
    rl = rl.reshape(steps, nb, nh)
    worst = 0.0
    for s in range(steps):
        assert_close(got_o[s], ro[s], dtype, "decode o, step %d (position %d)" % (s, ctx + s))
        assert_close(got_l[s], rl[s], dtype, "decode lse, step %d" % s)
        e = np.linalg.norm(got_o[s] - ro[s], axis=-1) / np.maximum(np.linalg.norm(ro[s], axis=-1), 1e-30)
        worst = max(worst, float(e.max()))
    assert worst < 5e-2, "worst (entry, head) row over all steps: rel err %.3g" % worst
    assert_close(got_sk, fk, dtype, "state_k after %d steps" % steps)
    assert_close(got_sv, fv, dtype, "state_v after %d steps" % steps)


@pytest.mark.parametrize("ctx", [4096, 16384, 32768])
def test_decode_workload_all_steps(ctx):
    # batch 256, H16 d128 D16: all 1024 steps, every step checked on 3 x 3 units
    w = wl.DECODE_D16
    long_decode_check(w, ctx, w.decode_steps, check_b=[0, 97, 255], check_h=[0, 5, 15], fill_chunk=16)


def test_hybrid_decode_workload_all_steps():
    # batch 128, 4 dense + 28 dilated/windowed heads: all 256 steps after the
    # 65536-token context, on entries spread over the full batch
    w = wl.HYBRID
    long_decode_check(w, 65536, w.decode_steps, check_b=[0, 63, 127], check_h=[0, 3, 4, 31], fill_chunk=4)

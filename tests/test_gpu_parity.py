"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Inputs come from workloads.py (seeded; q, k, v ~ N(0,1), gate logits ~ N(mu,1)).
The oracle consumes the exact input values the GPU consumed (bf16 inputs are
converted to fp64 on the host).  Bar: max-abs 1e-4 (fp32), relative L2 1e-2
(bf16).  Small cases compare every element; the full-size workloads compare
sampled heads and rows that always include t=0, t<D, residue and window
boundaries and the last rows.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import assert_close, f64, sample_rows

rat = pytest.importorskip("recurrence_augmented_dilated_gated_b200")

pytestmark = pytest.mark.gpu

DEV = "cuda"


def make_cfg(B, T, H, d, dtype, dil, win, recur=None, scale=0.0, grid=False, dedupe=False, sep=False, t0=0,
             t_cap=0):
    flags = (rat.RAT_FLAG_GRID_DILATION if grid else 0) | (rat.RAT_FLAG_DEDUPE if dedupe else 0)
    flags |= rat.RAT_FLAG_SEPARATE_GATES if sep else 0
    return rat.Config(B, T, H, d, dtype, dil, win, recur, scale, flags, t0, t_cap)


def inputs(B, T, H, d, dtype, mu=2.0, seed=0, device="cpu"):
    q, k, v, g = wl.prefill_inputs(B, T, H, d, mu, dtype, device=device, seed=seed)
    return [x.to(DEV) for x in (q, k, v, g)]


def oracle_prefill(q, k, v, g, dil, win, recur, init_k=None, init_v=None, scale=None):
    return oracle.mix_prefill(f64(q), f64(k), f64(v), f64(g), dil, win, recur,
                              None if init_k is None else f64(init_k), None if init_v is None else f64(init_v),
                              scale=scale)


# ------------------------------------------------------------------ small cases


def test_tiny_f32_operator_every_element():
    w = wl.TINY_F32
    cfg = make_cfg(w.B, w.T, w.H, w.d, rat.RAT_F32, w.dil, w.win, w.recur)
    q, k, v, g = inputs(w.B, w.T, w.H, w.d, torch.float32, w.gate_mean)
    out = rat.mix_prefill(cfg, q, k, v, g, want_kv=True)
    rat.rat_check_status(out["ws"])
    ref = oracle_prefill(q, k, v, g, w.dil, w.win, w.recur)
    for key in ("o", "lse", "kt", "vt", "final_k", "final_v"):
        assert_close(out[key], ref[key], torch.float32, key)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 77, 1000, 5003])
def test_scan_every_element(dtype, d, T):
    # ragged T spans one to dozens of chunks (look-back exercised); init given
    B, H = 2, 3
    q, k, v, g = inputs(B, T, H, d, dtype, seed=T)
    init_k = wl.random_state(B, H, d, seed=1).to(DEV)
    init_v = wl.random_state(B, H, d, seed=2).to(DEV)
    recur = [1, 0, 1]
    cfg = make_cfg(B, T, H, d, dtype, [4] * H, [0] * H, recur)
    kt, vt = torch.empty_like(k), torch.empty_like(v)
    fk = torch.empty(B, H, d, device=DEV)
    fv = torch.empty_like(fk)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_scan_prefill(cfg, k, v, g, init_k, init_v, kt, vt, fk, fv, ws=ws)
    rat.rat_check_status(ws)
    rk, rfk = oracle.scan(f64(k), f64(g), f64(init_k), recur)
    rv, rfv = oracle.scan(f64(v), f64(g), f64(init_v), recur)
    assert_close(kt, rk, dtype, "kt")
    assert_close(vt, rv, dtype, "vt")
    assert_close(fk, rfk, torch.float32 if dtype == torch.float32 else dtype, "final_k")
    assert_close(fv, rfv, torch.float32 if dtype == torch.float32 else dtype, "final_v")
    # heads without recurrence are copied exactly
    assert torch.equal(kt[:, :, 1], k[:, :, 1]) and torch.equal(vt[:, :, 1], v[:, :, 1])


ATTN_CASES = [
    # (T, dil per head, win per head)
    (700, [1, 3], [0, 0]),
    (700, [16, 5], [64, 1]),
    (333, [7, 400], [5, 333]),     # D > T for one head, W = T
    (129, [1, 2], [1000, 2]),      # W > T
    (1024, [64, 16], [512, 0]),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", range(len(ATTN_CASES)))
def test_attention_every_element(dtype, d, case):
    T, dil, win = ATTN_CASES[case]
    B, H = 2, 2
    q, kt, vt, _ = inputs(B, T, H, d, dtype, seed=100 + case)
    cfg = make_cfg(B, T, H, d, dtype, dil, win)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, T, device=DEV)
    ws = rat.workspace(cfg, rat.RAT_OP_ATTN)
    rat.rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse, ws)
    rat.rat_check_status(ws)
    ro, rl = oracle.attention(f64(q), f64(kt), f64(vt), dil, win)
    assert_close(o, ro, dtype, "o")
    assert_close(lse, rl, dtype if dtype == torch.bfloat16 else torch.float32, "lse")


TC_CASES = [
    # (B, T, dil per head, win per head): bf16 operands, so every head runs on
    # the tensor-core kernel; n = T/D spans full and partial 128-row tiles
    (2, 2048, [1, 4], [0, 0]),
    (2, 2048, [64, 1], [512, 100]),
    (1, 12800, [64, 64], [1, 3000]),       # n = 200: one full and one partial tile
    (2, 1000, [8, 1], [127, 128]),         # n = 125 < 128; window edges at tile size
    (1, 4096, [16, 2], [256, 4096]),
    # D not dividing T: the residues before T mod D have one row more; each of
    # the two groups runs through its own strided view, still on the tensor cores
    (2, 2000, [64, 3], [512, 0]),          # T mod D = 16 and 2
    (1, 12801, [64, 7], [1, 3000]),        # 201 / 200 and 1829 / 1828 rows per residue
    (2, 130, [400, 129], [0, 5]),          # D > T (130 one-row residues) and D = T - 1
    (1, 4097, [16, 1], [256, 0]),          # one residue of 257 rows, fifteen of 256
]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", range(len(TC_CASES)))
def test_tensor_core_attention_every_element(d, case):
    B, T, dil, win = TC_CASES[case]
    H = len(dil)
    dtype = torch.bfloat16
    q, kt, vt, _ = inputs(B, T, H, d, dtype, seed=300 + case)
    cfg = make_cfg(B, T, H, d, dtype, dil, win)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, T, device=DEV)
    ws = rat.workspace(cfg, rat.RAT_OP_ATTN)
    rat.rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse, ws)
    rat.rat_check_status(ws)
    ro, rl = oracle.attention(f64(q), f64(kt), f64(vt), dil, win)
    assert_close(o, ro, dtype, "o")
    assert_close(lse, rl, dtype, "lse")
    # every row, not only the bulk, within the bar: the worst row's relative error
    err = np.linalg.norm(f64(o) - ro, axis=-1) / np.maximum(np.linalg.norm(ro, axis=-1), 1e-30)
    assert float(err.max()) < 5e-2, "worst row rel err %.3g" % float(err.max())


def test_many_dilation_classes_split_over_launches():
    # 12 distinct dilations (more than one tensor-core launch holds) plus a
    # window on some heads; every head still matches the oracle
    B, T, d = 1, 2048, 64
    dil = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048] * 2
    win = [0] * 12 + [3, 0, 17, 0, 64, 0, 129, 0, 1, 0, 2048, 5]
    H = len(dil)
    dtype = torch.bfloat16
    q, kt, vt, _ = inputs(B, T, H, d, dtype, seed=400)
    cfg = make_cfg(B, T, H, d, dtype, dil, win)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, T, device=DEV)
    ws = rat.workspace(cfg, rat.RAT_OP_ATTN)
    rat.rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse, ws)
    rat.rat_check_status(ws)
    ro, rl = oracle.attention(f64(q), f64(kt), f64(vt), dil, win)
    for h in range(H):
        assert_close(o[:, :, h], ro[:, :, h], dtype, "o head %d (D=%d W=%d)" % (h, dil[h], win[h]))
    assert_close(lse, rl, dtype, "lse")


@pytest.mark.parametrize("T", [1, 2, 130])
def test_short_sequences_on_both_paths(T):
    # T = 1 (one row, one key), tiny T, and T just past one tile, for D | T
    # (tensor-core kernel) and D not dividing T (CUDA-core kernel)
    B, H, d = 2, 4, 128
    dil, win, recur = [1, 1, 3, T + 1], [0, 2, 1, 0], [0, 1, 1, 1]
    dtype = torch.bfloat16
    q, k, v, g = inputs(B, T, H, d, dtype, seed=500 + T)
    cfg = make_cfg(B, T, H, d, dtype, dil, win, recur)
    out = rat.mix_prefill(cfg, q, k, v, g, want_kv=True)
    rat.rat_check_status(out["ws"])
    ref = oracle_prefill(q, k, v, g, dil, win, recur)
    for key in ("o", "lse", "kt", "vt", "final_k", "final_v"):
        assert_close(out[key], ref[key], dtype, key)


def test_maximum_head_count():
    # H = 256, the largest head count the library accepts, mixed dilations
    B, T, H, d = 1, 64, 256, 64
    dil = [1 + (h % 4) for h in range(H)]
    win = [(h % 3) * 4 for h in range(H)]
    dtype = torch.bfloat16
    q, k, v, g = inputs(B, T, H, d, dtype, seed=600)
    cfg = make_cfg(B, T, H, d, dtype, dil, win)
    out = rat.mix_prefill(cfg, q, k, v, g)
    rat.rat_check_status(out["ws"])
    ref = oracle_prefill(q, k, v, g, dil, win, None)
    assert_close(out["o"], ref["o"], dtype, "o")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mix_hybrid_heads_every_element(dtype):
    # dense heads (D=1, no recurrence) next to dilated + windowed recurrent heads
    B, T, H, d = 2, 960, 4, 128
    dil, win, recur = [1, 1, 8, 7], [0, 0, 32, 100], [0, 0, 1, 1]   # 7 does not divide 960: CUDA-core path
    q, k, v, g = inputs(B, T, H, d, dtype, mu=3.0, seed=7)
    init_k = wl.random_state(B, H, d, seed=3).to(DEV)
    cfg = make_cfg(B, T, H, d, dtype, dil, win, recur)
    for want_kv in (False, True):
        out = rat.mix_prefill(cfg, q, k, v, g, init_k=init_k, want_kv=want_kv)
        rat.rat_check_status(out["ws"])
        ref = oracle_prefill(q, k, v, g, dil, win, recur, init_k=init_k)
        assert_close(out["o"], ref["o"], dtype, "o")
        assert_close(out["lse"], ref["lse"], torch.float32 if dtype == torch.float32 else dtype, "lse")
        ft = torch.float32 if dtype == torch.float32 else dtype
        assert_close(out["final_k"], ref["final_k"], ft, "final_k")
        assert_close(out["final_v"], ref["final_v"], ft, "final_v")
        if want_kv:
            assert_close(out["kt"], ref["kt"], dtype, "kt")


def test_custom_scale():
    B, T, H, d = 1, 300, 2, 64
    dtype = torch.bfloat16
    q, k, v, g = inputs(B, T, H, d, dtype, seed=11)
    cfg = make_cfg(B, T, H, d, dtype, [3, 3], [10, 0], scale=0.05)
    out = rat.mix_prefill(cfg, q, k, v, g)
    ref = oracle_prefill(q, k, v, g, [3, 3], [10, 0], None, scale=0.05)
    assert_close(out["o"], ref["o"], dtype, "o")


def test_empty_inputs():
    B, T, H, d = 2, 0, 2, 64
    cfg = make_cfg(B, T, H, d, torch.float32, [2, 2], [0, 0])
    e = torch.empty(B, T, H, d, device=DEV)
    init = wl.random_state(B, H, d, seed=5).to(DEV)
    fk = torch.full((B, H, d), 7.0, device=DEV)
    fv = torch.full((B, H, d), 7.0, device=DEV)
    ws = rat.workspace(make_cfg(B, 1, H, d, torch.float32, [2, 2], [0, 0]), rat.RAT_OP_MIX)
    rat.rat_mix_prefill(cfg, e, e, e, e, init, None, e, None, None, None, fk, fv, ws)
    torch.cuda.synchronize()
    assert torch.equal(fk, init) and torch.all(fv == 0)


def test_workspace_reused_across_calls():
    # one workspace for several calls with different inputs: the per-call
    # reset of the attention work counters and of the scan's chunk flags
    B, T, H, d, dtype = 1, 2048, 3, 128, torch.bfloat16
    dil, win, recur = [16, 1, 4], [128, 0, 0], [1, 0, 1]
    cfg = make_cfg(B, T, H, d, dtype, dil, win, recur)
    ws = rat.workspace(cfg, rat.RAT_OP_MIX)
    o = torch.empty(B, T, H, d, dtype=dtype, device=DEV)
    lse = torch.empty(B, H, T, device=DEV)
    for call in range(3):
        q, k, v, g = inputs(B, T, H, d, dtype, seed=900 + call)
        rat.rat_mix_prefill(cfg, q, k, v, g, None, None, o, lse, None, None, None, None, ws)
        rat.rat_check_status(ws)
        kt, _ = oracle.scan(f64(k), f64(g), None, recur)
        vt, _ = oracle.scan(f64(v), f64(g), None, recur)
        ro, rl = oracle.attention(f64(q), kt, vt, dil, win)
        assert_close(o, ro, dtype, "o, call %d" % call)
        assert_close(lse, rl, dtype, "lse, call %d" % call)


def test_decode_cache_layout_from_scan():
    # cache row of position j in head h: (j mod D_h) * ceil(cap/D_h) + j // D_h
    B, T, H, d = 2, 300, 3, 64
    dtype = torch.bfloat16
    dil = [1, 4, 7]
    cap = 333
    q, k, v, g = inputs(B, T, H, d, dtype, seed=9)
    cfg = make_cfg(B, T, H, d, dtype, dil, [0] * H)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    kt, vt = torch.empty_like(k), torch.empty_like(v)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_scan_prefill(cfg, k, v, g, None, None, kt, vt, None, None, ck, cv, cap, ws)
    torch.cuda.synchronize()
    for h, D in enumerate(dil):
        S = -(-cap // D)
        j = torch.arange(T, device=DEV)
        rows = (j % D) * S + j // D
        assert torch.equal(ck[:, h, rows], kt[:, :, h])
        assert torch.equal(cv[:, h, rows], vt[:, :, h])


def run_decode_case(B, T, steps, H, d, dtype, dil, win, recur, mu, seed, cap=None, check_b=None, check_h=None,
                    gen_device="cpu", grid=False, dedupe=False, sep=False):
    """Prefill T tokens into the cache with rat_scan_prefill, then decode `steps`
    tokens with rat_decode_step; compare every step with the oracle's rows
    (on the batch entries check_b and heads check_h; all by default).  grid:
    the fixed-grid reading of dilation and its cache layout; dedupe: a key in
    both parts counts once; sep: separate key and value gates."""
    Tt = T + steps
    cap = cap or Tt
    q, k, v, g = inputs(B, Tt, H, d, dtype, mu=mu, seed=seed, device=gen_device)
    gv = inputs(B, Tt, H, d, dtype, mu=mu, seed=seed + 1000, device=gen_device)[3] if sep else g
    cfg = make_cfg(B, T, H, d, dtype, dil, win, recur, grid=grid, dedupe=dedupe, sep=sep)
    # the gate argument: [2, B, T, H, d] with separate gates
    gate = (lambda sl: torch.stack([g[sl], gv[sl]]).contiguous()) if sep else (lambda sl: g[sl].contiguous())
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    sk = torch.empty(B, H, d, device=DEV)
    sv = torch.empty_like(sk)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_scan_prefill(cfg, k[:, :T].contiguous(), v[:, :T].contiguous(), gate(np.s_[:, :T]), None, None,
                         None, None, sk, sv, ck, cv, cap, ws)
    rat.rat_check_status(ws)
    del ws
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    outs = []
    for s in range(steps):
        t = T + s
        pos = torch.full((B,), t, dtype=torch.int32, device=DEV)
        o = torch.empty(B, H, d, dtype=dtype, device=DEV)
        lse = torch.empty(B, H, device=DEV)
        rat.rat_decode_step(cfg, q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                            gate(np.s_[:, t]), sk, sv, ck, cv, cap, pos, o, lse, wsd)
        outs.append((o, lse))
    rat.rat_check_status(wsd)
    bsel = list(range(B)) if check_b is None else check_b
    hsel = list(range(H)) if check_h is None else check_h
    sl = lambda x: f64(x[bsel][:, :, hsel])
    dsel, wsel, rsel = [dil[h] for h in hsel], [win[h] for h in hsel], [recur[h] for h in hsel]
    kt, fk = oracle.scan(sl(k), sl(g), None, rsel)
    vt, fv = oracle.scan(sl(v), sl(gv), None, rsel)
    rows = np.array([(b, i, t) for b in range(len(bsel)) for i in range(len(hsel)) for t in range(T, Tt)])
    ro, rl = oracle.attn_rows(sl(q), kt, vt, dsel, wsel, rows, parts=3, grid=grid, dedupe=dedupe)
    ro = ro.reshape(len(bsel), len(hsel), steps, d)
    rl = rl.reshape(len(bsel), len(hsel), steps)
    ft = torch.float32 if dtype == torch.float32 else dtype
    for s, (o, lse) in enumerate(outs):
        assert_close(o[bsel][:, hsel], ro[:, :, s], dtype, "decode o step %d" % s)
        assert_close(lse[bsel][:, hsel], rl[:, :, s], ft, "decode lse step %d" % s)
    assert_close(sk[bsel][:, hsel], fk, ft, "state_k")
    assert_close(sv[bsel][:, hsel], fv, ft, "state_v")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_steps_every_element(dtype, d):
    run_decode_case(B=3, T=1500, steps=5, H=4, d=d, dtype=dtype, dil=[1, 4, 16, 3], win=[0, 0, 64, 1500],
                    recur=[0, 1, 1, 1], mu=2.0, seed=21)


def test_decode_from_empty_history():
    # the first token decoded with nothing in the cache (t = 0), then a few more
    run_decode_case(B=2, T=1, steps=4, H=2, d=128, dtype=torch.bfloat16, dil=[2, 1], win=[3, 0],
                    recur=[1, 0], mu=2.0, seed=5, cap=8)


def test_decode_long_slab_spans_several_splits():
    # 2500 old rows in the residue slab: at batch 1 the plan splits it into ten
    # 256-row items (the last one also does the step update), combined by LSE
    run_decode_case(B=1, T=5000, steps=2, H=2, d=128, dtype=torch.bfloat16, dil=[2, 1], win=[0, 7],
                    recur=[1, 1], mu=2.0, seed=6)


def _prefill_cache_per_entry(cfg1, k, v, g, T_b, cap, ck, cv, sk, sv):
    """Fill batch entry b's cache rows and state from its own T_b tokens (one
    B = 1 scan per entry, writing into that entry's slices)."""
    for b, Tb in enumerate(T_b):
        c = cfg1.replace(B=1, T=Tb)
        ws = rat.workspace(c, rat.RAT_OP_SCAN)
        rat.rat_scan_prefill(c, k[b:b + 1, :Tb].contiguous(), v[b:b + 1, :Tb].contiguous(),
                             g[b:b + 1, :Tb].contiguous(), None, None, None, None, sk[b:b + 1], sv[b:b + 1],
                             ck[b:b + 1], cv[b:b + 1], cap, ws)
        rat.rat_check_status(ws)


def test_decode_ragged_positions():
    # each sequence of the batch at its own position (pos is per entry): a
    # batch entry reads only its own residue slab and window
    B, H, d, dtype = 4, 3, 128, torch.bfloat16
    dil, win, recur = [1, 8, 5], [0, 16, 33], [0, 1, 1]
    T_b = [1, 700, 1299, 2048]
    steps, cap = 3, max(T_b) + 3
    Tt = max(T_b) + steps
    q, k, v, g = inputs(B, Tt, H, d, dtype, seed=31)
    cfg = make_cfg(B, max(T_b), H, d, dtype, dil, win, recur)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    sk = torch.empty(B, H, d, device=DEV)
    sv = torch.empty_like(sk)
    _prefill_cache_per_entry(cfg, k, v, g, T_b, cap, ck, cv, sk, sv)
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    kt, _ = oracle.scan(f64(k), f64(g), None, recur)
    vt, _ = oracle.scan(f64(v), f64(g), None, recur)
    for s in range(steps):
        pos_l = [t + s for t in T_b]
        pos = torch.tensor(pos_l, dtype=torch.int32, device=DEV)
        tok = lambda x: torch.stack([x[b, pos_l[b]] for b in range(B)]).contiguous()
        o = torch.empty(B, H, d, dtype=dtype, device=DEV)
        lse = torch.empty(B, H, device=DEV)
        rat.rat_decode_step(cfg, tok(q), tok(k), tok(v), tok(g), sk, sv, ck, cv, cap, pos, o, lse, wsd)
        rows = np.array([(b, h, pos_l[b]) for b in range(B) for h in range(H)])
        ro, rl = oracle.attn_rows(f64(q), kt, vt, dil, win, rows, parts=3)
        assert_close(o, ro.reshape(B, H, d), dtype, "ragged decode o step %d" % s)
        assert_close(lse, rl.reshape(B, H), torch.float32 if dtype == torch.float32 else dtype,
                     "ragged decode lse step %d" % s)
    rat.rat_check_status(wsd)


def test_decode_step_replays_from_a_cuda_graph():
    # one rat_decode_step captured in a CUDA graph (its counter reset and its
    # kernel), replayed for several tokens with the inputs and positions
    # refreshed in place between replays
    B, H, d, dtype = 2, 2, 128, torch.bfloat16
    dil, win, recur = [4, 1], [8, 0], [1, 0]
    T, steps = 1000, 4
    cap = T + steps
    q, k, v, g = inputs(B, T + steps, H, d, dtype, seed=41)
    cfg = make_cfg(B, T, H, d, dtype, dil, win, recur)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    sk = torch.empty(B, H, d, device=DEV)
    sv = torch.empty_like(sk)
    _prefill_cache_per_entry(cfg, k, v, g, [T] * B, cap, ck, cv, sk, sv)
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    xq, xk, xv, xg = (torch.empty(B, H, d, dtype=dtype, device=DEV) for _ in range(4))
    pos = torch.full((B,), T, dtype=torch.int32, device=DEV)
    o = torch.empty(B, H, d, dtype=dtype, device=DEV)
    lse = torch.empty(B, H, device=DEV)
    # a first eager step (also warms up), then capture the same step
    for x_, src in zip((xq, xk, xv, xg), (q, k, v, g)):
        x_.copy_(src[:, T])
    rat.rat_decode_step(cfg, xq, xk, xv, xg, sk, sv, ck, cv, cap, pos, o, lse, wsd)
    torch.cuda.synchronize()
    outs = [(o.clone(), lse.clone())]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        rat.rat_decode_step(cfg, xq, xk, xv, xg, sk, sv, ck, cv, cap, pos, o, lse, wsd)
    for s in range(1, steps):
        for x_, src in zip((xq, xk, xv, xg), (q, k, v, g)):
            x_.copy_(src[:, T + s])
        pos.fill_(T + s)
        graph.replay()
        outs.append((o.clone(), lse.clone()))
    torch.cuda.synchronize()
    rat.rat_check_status(wsd)
    kt, fk = oracle.scan(f64(k), f64(g), None, recur)
    vt, fv = oracle.scan(f64(v), f64(g), None, recur)
    rows = np.array([(b, h, t) for b in range(B) for h in range(H) for t in range(T, T + steps)])
    ro, rl = oracle.attn_rows(f64(q), kt, vt, dil, win, rows, parts=3)
    ro = ro.reshape(B, H, steps, d)
    rl = rl.reshape(B, H, steps)
    for s, (os_, ls_) in enumerate(outs):
        assert_close(os_, ro[:, :, s], dtype, "graph decode o step %d" % s)
        assert_close(ls_, rl[:, :, s], dtype, "graph decode lse step %d" % s)
    assert_close(sk, fk, dtype, "state_k after the replays")
    assert_close(sv, fv, dtype, "state_v after the replays")
    del graph


# ------------------------------------------------- fixed-grid reading of dilation
# Query t attends to { j <= t : j mod D == D-1 } plus itself, and the decode
# cache keeps only the grid rows plus a ring of the last W positions.

GRID_CASES = [
    # (B, T, dil per head, win per head)
    (2, 2048, [4, 64], [0, 100]),        # tensor-core grid launch, one head windowed
    (1, 12800, [64, 128], [1, 3000]),    # 200 and 100 grid rows: full and partial key tiles
    (2, 1024, [256, 1], [0, 64]),        # D = 256: the first query tiles have no grid key yet
    (2, 1000, [8, 3], [127, 0]),         # 3 does not divide T: the grid is 333 rows of residue 2
    (1, 5003, [64, 7], [512, 0]),        # T mod D = 11 and 5: ragged grids on the tensor cores
    (2, 100, [128, 101], [0, 7]),        # D > T: no grid key anywhere, every row attends to itself
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", range(len(GRID_CASES)))
def test_grid_attention_every_element(dtype, d, case):
    B, T, dil, win = GRID_CASES[case]
    H = len(dil)
    q, kt, vt, _ = inputs(B, T, H, d, dtype, seed=700 + case)
    cfg = make_cfg(B, T, H, d, dtype, dil, win, grid=True)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, T, device=DEV)
    ws = rat.workspace(cfg, rat.RAT_OP_ATTN)
    rat.rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse, ws)
    rat.rat_check_status(ws)
    ro, rl = oracle.attention(f64(q), f64(kt), f64(vt), dil, win, grid=True)
    assert_close(o, ro, dtype, "o")
    assert_close(lse, rl, dtype if dtype == torch.bfloat16 else torch.float32, "lse")
    err = np.linalg.norm(f64(o) - ro, axis=-1) / np.maximum(np.linalg.norm(ro, axis=-1), 1e-30)
    assert float(err.max()) < 5e-2, "worst row rel err %.3g" % float(err.max())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_grid_mix_hybrid_heads_every_element(dtype):
    # a dense head without recurrence next to dilated recurrent heads
    B, T, d = 2, 1536, 128
    dil, win, recur = [1, 16, 64], [0, 0, 256], [0, 1, 1]
    H = len(dil)
    q, k, v, g = inputs(B, T, H, d, dtype, seed=77)
    cfg = make_cfg(B, T, H, d, dtype, dil, win, recur, grid=True)
    out = rat.mix_prefill(cfg, q, k, v, g)
    rat.rat_check_status(out["ws"])
    rk, _ = oracle.scan(f64(k), f64(g), None, recur)
    rv, _ = oracle.scan(f64(v), f64(g), None, recur)
    ro, rl = oracle.attention(f64(q), rk, rv, dil, win, grid=True)
    assert_close(out["o"], ro, dtype, "o")
    assert_close(out["lse"], rl, dtype if dtype == torch.bfloat16 else torch.float32, "lse")


def test_grid_decode_cache_layout_from_scan():
    # grid row of j (j mod D == D-1): j // D; ring row (D > 1, W > 0) of the
    # prefill's last W positions: ceil(cap / D) + j mod W
    B, T, H, d = 2, 300, 4, 64
    dtype = torch.bfloat16
    dil, win = [1, 4, 7, 16], [5, 0, 40, 512]
    cap = 333
    q, k, v, g = inputs(B, T, H, d, dtype, seed=19)
    cfg = make_cfg(B, T, H, d, dtype, dil, win, grid=True)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    kt, vt = torch.empty_like(k), torch.empty_like(v)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_scan_prefill(cfg, k, v, g, None, None, kt, vt, None, None, ck, cv, cap, ws)
    rat.rat_check_status(ws)
    for h, (D, W) in enumerate(zip(dil, win)):
        S = -(-cap // D)
        j = torch.arange(D - 1, T, D, device=DEV)
        assert torch.equal(ck[:, h, j // D], kt[:, j, h])
        assert torch.equal(cv[:, h, j // D], vt[:, j, h])
        if D > 1 and W > 0:
            j = torch.arange(max(0, T - W), T, device=DEV)
            assert torch.equal(ck[:, h, S + j % W], kt[:, j, h])
            assert torch.equal(cv[:, h, S + j % W], vt[:, j, h])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_grid_decode_steps_every_element(dtype, d):
    # positions 1500..1504 put t on the grid of D = 4, 16 and 3 once each
    run_decode_case(B=3, T=1500, steps=5, H=4, d=d, dtype=dtype, dil=[1, 4, 16, 3], win=[0, 0, 64, 1500],
                    recur=[0, 1, 1, 1], mu=2.0, seed=21, grid=True)


def test_grid_decode_from_empty_history():
    # the ring fills while the first positions are decoded (cap 8 < W for one head)
    run_decode_case(B=2, T=1, steps=6, H=3, d=128, dtype=torch.bfloat16, dil=[2, 1, 3], win=[3, 0, 10],
                    recur=[1, 0, 1], mu=2.0, seed=5, cap=8, grid=True)


def test_grid_decode_long_slab_spans_several_splits():
    run_decode_case(B=1, T=5000, steps=2, H=2, d=128, dtype=torch.bfloat16, dil=[2, 1], win=[9, 7],
                    recur=[1, 1], mu=2.0, seed=6, grid=True)


# ------------------------------------------------- dedupe: a shared key counts once

DEDUPE_CASES = [
    # (B, T, dil per head, win per head): windows wider and narrower than D
    (2, 2048, [4, 64], [100, 512]),
    (1, 1056, [1, 33], [64, 1000]),       # D = 1: no window part; D = 33 > 32 (one key per chunk)
    (2, 768, [2, 3], [1, 300]),           # W = 1 leaves the window part empty (residue reading)
    (2, 1000, [8, 7], [127, 50]),         # 7 does not divide T: CUDA cores
]


@pytest.mark.parametrize("grid", [False, True])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("case", range(len(DEDUPE_CASES)))
def test_dedupe_attention_every_element(grid, dtype, case):
    B, T, dil, win = DEDUPE_CASES[case]
    H, d = len(dil), 128
    q, kt, vt, _ = inputs(B, T, H, d, dtype, seed=900 + case)
    cfg = make_cfg(B, T, H, d, dtype, dil, win, grid=grid, dedupe=True)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, T, device=DEV)
    ws = rat.workspace(cfg, rat.RAT_OP_ATTN)
    rat.rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse, ws)
    rat.rat_check_status(ws)
    ro, rl = oracle.attention(f64(q), f64(kt), f64(vt), dil, win, grid=grid, dedupe=True)
    assert_close(o, ro, dtype, "o")
    assert_close(lse, rl, dtype if dtype == torch.bfloat16 else torch.float32, "lse")
    err = np.linalg.norm(f64(o) - ro, axis=-1) / np.maximum(np.linalg.norm(ro, axis=-1), 1e-30)
    assert float(err.max()) < 5e-2, "worst row rel err %.3g" % float(err.max())


@pytest.mark.parametrize("grid", [False, True])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dedupe_decode_steps_every_element(grid, dtype):
    run_decode_case(B=3, T=1500, steps=5, H=4, d=128, dtype=dtype, dil=[1, 4, 16, 3], win=[8, 9, 64, 1500],
                    recur=[0, 1, 1, 1], mu=2.0, seed=23, grid=grid, dedupe=True)


# ------------------------------------------- top-k block attention for decoding


def run_topk_case(B, T, steps, H, d, dtype, block, topk, mode, recur, seed, cap=None, margin=0.02):
    """Prefill T tokens into a dense cache, build the block statistics, decode
    `steps` tokens with rat_topk_decode_step; compare with the oracle's top-k
    rows.  The block choice is an integer decision: the oracle takes it on its
    K~ rounded to the cache's precision, as the kernel does, and rows whose
    K-th and (K+1)-th block scores lie within `margin` (rounding could swap
    them) are only checked for a valid selection."""
    Tt = T + steps
    cap = cap or Tt
    q, k, v, g = inputs(B, Tt, H, d, dtype, mu=2.0, seed=seed)
    cfg = make_cfg(B, T, H, d, dtype, [1] * H, [0] * H, recur)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    sk = torch.empty(B, H, d, device=DEV)
    sv = torch.empty_like(sk)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_scan_prefill(cfg, k[:, :T].contiguous(), v[:, :T].contiguous(), g[:, :T].contiguous(), None, None,
                         None, None, sk, sv, ck, cv, cap, ws)
    rat.rat_check_status(ws)
    stats = torch.full(rat.topk_stats_shape(cfg, block, cap), float("nan"), device=DEV)
    rat.rat_topk_build_stats(cfg, block, mode, ck, cap, stats)
    wsd = rat.workspace(cfg, rat.RAT_OP_TOPK_DECODE, cap)
    outs = []
    for s in range(steps):
        t = T + s
        pos = torch.full((B,), t, dtype=torch.int32, device=DEV)
        o = torch.empty(B, H, d, dtype=dtype, device=DEV)
        lse = torch.empty(B, H, device=DEV)
        sel = torch.empty(B, H, topk, dtype=torch.int32, device=DEV)
        rat.rat_topk_decode_step(cfg, block, topk, mode, q[:, t].contiguous(), k[:, t].contiguous(),
                                 v[:, t].contiguous(), g[:, t].contiguous(), sk, sv, ck, cv, cap, stats, pos, o,
                                 lse, sel, wsd)
        outs.append((o, lse, sel))
    rat.rat_check_status(wsd)
    kt, fk = oracle.scan(f64(k), f64(g), None, recur)
    vt, fv = oracle.scan(f64(v), f64(g), None, recur)
    ft = torch.float32 if dtype == torch.float32 else dtype
    assert_close(ck[:, :, :Tt].transpose(1, 2), kt, dtype, "cache_k")
    assert_close(cv[:, :, :Tt].transpose(1, 2), vt, dtype, "cache_v")
    assert_close(sk, fk, ft, "state_k")
    # the cache's precision for the oracle's keys and values
    kq = torch.from_numpy(kt).to(dtype).double().numpy()
    vq = torch.from_numpy(vt).to(dtype).double().numpy()
    name = {rat.RAT_TOPK_QUEST: "quest", rat.RAT_TOPK_MOBA: "moba"}[mode]
    rows = np.array([(b, h, t) for b in range(B) for h in range(H) for t in range(T, Tt)])
    ro, rl = oracle.attn_rows_topk(f64(q), kq, vq, block, topk, name, rows)
    rsel, gap = oracle.topk_select(f64(q), kq, block, topk, name, rows)
    got_o = np.stack([f64(o) for o, _, _ in outs], axis=2).reshape(-1, d)      # (b, h, step) order
    got_l = np.stack([f64(l) for _, l, _ in outs], axis=2).reshape(-1)
    got_s = np.stack([x[2].cpu().numpy() for x in outs], axis=2).reshape(-1, topk)
    clear = gap > margin
    assert clear.mean() >= 0.6, "too many near-ties: %d of %d rows" % (int((~clear).sum()), len(clear))
    for i in np.nonzero(clear)[0]:
        assert sorted(got_s[i]) == sorted(rsel[i]), (rows[i], got_s[i], rsel[i])
    assert_close(got_o[clear], ro[clear], dtype, "top-k o")
    assert_close(got_l[clear], rl[clear], ft, "top-k lse")
    for i in np.nonzero(~clear)[0]:   # a near-tie: any valid selection of distinct candidates
        c = rows[i][2] // block
        picked = [x for x in got_s[i] if x >= 0]
        assert len(set(picked)) == len(picked) == min(topk, max(0, c - 1))
        assert all(1 <= x < c for x in picked)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_topk_decode_steps(mode, dtype, d):
    # positions 1021 .. 1025 cross into a new 64-row block at 1024
    run_topk_case(B=2, T=1021, steps=5, H=3, d=d, dtype=dtype, block=64, topk=4, mode=mode, recur=[0, 1, 1],
                  seed=31 + mode)


@pytest.mark.parametrize("mode", [0, 1])
def test_topk_decode_from_empty_history(mode):
    # blocks of 4 from t = 1: no candidates, then fewer than K, then more
    run_topk_case(B=2, T=1, steps=30, H=2, d=128, dtype=torch.bfloat16, block=4, topk=3, mode=mode,
                  recur=[1, 0], seed=41, cap=40)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("d,block,dtype", [(128, 37, torch.bfloat16), (128, 100, torch.bfloat16),
                                           (64, 37, torch.bfloat16), (128, 37, torch.float32)])
def test_topk_decode_many_candidates_odd_blocks(mode, d, block, dtype):
    # more candidates than one shared-memory chunk of statistics holds (16 per
    # chunk at d = 128, 32 at d = 64: 19 to 53 here), and blocks whose rows are
    # not a multiple of the row chunk (32 bf16 rows at d = 128, 16 fp32 rows,
    # 64 bf16 rows at d = 64), so both streams wrap their double buffer and
    # row groups realign at every block
    run_topk_case(B=2, T=2000, steps=3, H=2, d=d, dtype=dtype, block=block, topk=8, mode=mode, recur=[1, 1],
                  seed=47 + mode)


def test_topk_decode_keeps_every_block_when_k_is_large():
    # K >= number of candidates: the step is dense causal attention
    run_topk_case(B=1, T=500, steps=3, H=2, d=128, dtype=torch.bfloat16, block=32, topk=64, mode=0,
                  recur=[1, 1], seed=43)


# ------------------------------------------------- separate key and value gates


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [77, 5003])
def test_separate_gates_scan_every_element(dtype, d, T):
    B, H = 2, 3
    q, k, v, g = inputs(B, T, H, d, dtype, seed=T + 1)
    gv = inputs(B, T, H, d, dtype, mu=0.5, seed=T + 2)[3]
    init_k = wl.random_state(B, H, d, seed=3).to(DEV)
    init_v = wl.random_state(B, H, d, seed=4).to(DEV)
    recur = [1, 0, 1]
    cap = T + 5
    cfg = make_cfg(B, T, H, d, dtype, [1, 4, 7], [0, 0, 9], recur, sep=True)
    kt, vt = torch.empty_like(k), torch.empty_like(v)
    fk = torch.empty(B, H, d, device=DEV)
    fv = torch.empty_like(fk)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_scan_prefill(cfg, k, v, torch.stack([g, gv]).contiguous(), init_k, init_v, kt, vt, fk, fv, ck, cv,
                         cap, ws)
    rat.rat_check_status(ws)
    rk, rfk = oracle.scan(f64(k), f64(g), f64(init_k), recur)
    rv, rfv = oracle.scan(f64(v), f64(gv), f64(init_v), recur)
    ft = torch.float32 if dtype == torch.float32 else dtype
    assert_close(kt, rk, dtype, "kt")
    assert_close(vt, rv, dtype, "vt")
    assert_close(fk, rfk, ft, "final_k")
    assert_close(fv, rfv, ft, "final_v")
    for h, D in enumerate([1, 4, 7]):   # both caches written, each from its own pass
        S = -(-cap // D)
        j = torch.arange(T, device=DEV)
        rows = (j % D) * S + j // D
        assert torch.equal(ck[:, h, rows], kt[:, :, h]) and torch.equal(cv[:, h, rows], vt[:, :, h])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_separate_gates_mix_every_element(dtype):
    B, T, H, d = 2, 2048, 3, 128
    dil, win, recur = [1, 16, 64], [0, 0, 256], [0, 1, 1]
    q, k, v, g = inputs(B, T, H, d, dtype, seed=51)
    gv = inputs(B, T, H, d, dtype, mu=-1.0, seed=52)[3]
    cfg = make_cfg(B, T, H, d, dtype, dil, win, recur, sep=True)
    out = rat.mix_prefill(cfg, q, k, v, torch.stack([g, gv]).contiguous())
    rat.rat_check_status(out["ws"])
    rk, rfk = oracle.scan(f64(k), f64(g), None, recur)
    rv, rfv = oracle.scan(f64(v), f64(gv), None, recur)
    ro, rl = oracle.attention(f64(q), rk, rv, dil, win)
    ft = torch.float32 if dtype == torch.float32 else dtype
    assert_close(out["o"], ro, dtype, "o")
    assert_close(out["lse"], rl, ft, "lse")
    assert_close(out["final_k"], rfk, ft, "final_k")
    assert_close(out["final_v"], rfv, ft, "final_v")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_separate_gates_decode_steps(dtype):
    run_decode_case(B=3, T=1500, steps=4, H=4, d=128, dtype=dtype, dil=[1, 4, 16, 3], win=[0, 0, 64, 1500],
                    recur=[0, 1, 1, 1], mu=2.0, seed=25, sep=True)


# ---------------------------------------------------------- paged decode cache


def _paged_setup(grid):
    B, T, steps, H, d = 3, 700, 4, 3, 128
    dil, win, recur = [1, 4, 7], [0, 16, 100], [0, 1, 1]
    cap = T + steps
    dtype = torch.bfloat16
    q, k, v, g = inputs(B, T + steps, H, d, dtype, seed=61)
    cfg = make_cfg(B, T, H, d, dtype, dil, win, recur, grid=grid)
    R = rat.rat_cache_rows(cfg, cap)
    P = 48                      # not a multiple of a ring stage (64 rows): stages straddle pages
    pps = -(-R // P)
    num_pages = B * pps + 5
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(7))[:B * pps]
    table = perm.view(B, pps).to(torch.int32).to(DEV)
    return B, T, steps, H, d, cap, dtype, q, k, v, g, cfg, R, P, num_pages, table


@pytest.mark.parametrize("grid", [False, True])
def test_paged_decode_equals_dense(grid):
    # the same logical rows in shuffled pages: every output bit-identical
    B, T, steps, H, d, cap, dtype, q, k, v, g, cfg, R, P, num_pages, table = _paged_setup(grid)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    pool_k = torch.zeros(num_pages, H, P, d, dtype=dtype, device=DEV)
    pool_v = torch.zeros_like(pool_k)
    cache = rat.paged_cache(cfg, pool_k, pool_v, table, cap)
    states = [torch.empty(B, H, d, device=DEV) for _ in range(4)]
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    pre = (k[:, :T].contiguous(), v[:, :T].contiguous(), g[:, :T].contiguous())
    rat.rat_scan_prefill(cfg, *pre, None, None, None, None, states[0], states[1], ck, cv, cap, ws)
    rat.rat_scan_prefill_paged(cfg, *pre, None, None, None, None, states[2], states[3], cache=cache, cache_cap=cap,
                               ws=ws)
    rat.rat_check_status(ws)
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    for s in range(steps):
        t = T + s
        pos = torch.full((B,), t, dtype=torch.int32, device=DEV)
        tok = (q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), g[:, t].contiguous())
        o1, o2 = torch.empty(B, H, d, dtype=dtype, device=DEV), torch.empty(B, H, d, dtype=dtype, device=DEV)
        l1, l2 = torch.empty(B, H, device=DEV), torch.empty(B, H, device=DEV)
        rat.rat_decode_step(cfg, *tok, states[0], states[1], ck, cv, cap, pos, o1, l1, wsd)
        rat.rat_decode_step_paged(cfg, *tok, states[2], states[3], cache, cap, pos, o2, l2, wsd)
        rat.rat_check_status(wsd)
        assert torch.equal(o1, o2) and torch.equal(l1, l2), "step %d" % s
    assert torch.equal(states[0], states[2]) and torch.equal(states[1], states[3])
    # every logical row sits in the page the table names
    r = torch.arange(R, device=DEV)
    for b in range(B):
        pg = table[b, r // P].long()
        for h in range(H):
            assert torch.equal(pool_k[pg, h, r % P], ck[b, h]) and torch.equal(pool_v[pg, h, r % P], cv[b, h])


def test_paged_decode_invalid_page_is_reported():
    # a table entry of -1 on a page the step reads: every head of entry 1 reads
    # logical rows from 0 at t = 700 (residue 0 of D = 1, 4, 7), so all are
    # skipped (o = 0) and RAT_ERR_INVALID recorded; the other entries are not
    B, T, steps, H, d, cap, dtype, q, k, v, g, cfg, R, P, num_pages, table = _paged_setup(False)
    pool_k = torch.zeros(num_pages, H, P, d, dtype=dtype, device=DEV)
    pool_v = torch.zeros_like(pool_k)
    cache = rat.paged_cache(cfg, pool_k, pool_v, table, cap)
    sk, sv = torch.empty(B, H, d, device=DEV), torch.empty(B, H, d, device=DEV)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_scan_prefill_paged(cfg, k[:, :T].contiguous(), v[:, :T].contiguous(), g[:, :T].contiguous(), None,
                               None, None, None, sk, sv, cache=cache, cache_cap=cap, ws=ws)
    rat.rat_check_status(ws)
    ok = table.clone()
    table[1, 0] = -1            # head 0 of entry 1 (D = 1) reads logical rows from 0
    t = T
    pos = torch.full((B,), t, dtype=torch.int32, device=DEV)
    o = torch.empty(B, H, d, dtype=dtype, device=DEV)
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    rat.rat_decode_step_paged(cfg, q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                              g[:, t].contiguous(), sk, sv, cache, cap, pos, o, None, wsd)
    with pytest.raises(rat.RatError) as err:
        rat.rat_check_status(wsd)
    assert err.value.status == rat.RAT_ERR_INVALID
    assert torch.count_nonzero(o[1]) == 0
    assert torch.count_nonzero(o[0]) > 0 and torch.count_nonzero(o[2]) > 0
    table.copy_(ok)


# ------------------------------------------------------------- chunked prefill


@pytest.mark.parametrize("grid", [False, True])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("chunks", [[1024, 512, 448], [1000, 600, 384]])
def test_chunked_prefill_equals_one_shot(grid, dtype, chunks):
    # the chunks carry the recurrent state and share one kt/vt history buffer
    # (t_cap rows per batch entry); the second chunk list starts chunks at
    # 1000 and 1600, which D = 64 does not divide (those heads run on CUDA cores)
    B, H, d = 2, 3, 128
    dil, win, recur = [1, 8, 64], [0, 32, 300], [0, 1, 1]
    Ttot = sum(chunks)
    cap = Ttot + 8
    q, k, v, g = inputs(B, Ttot, H, d, dtype, seed=81)
    kt = torch.zeros(B, cap, H, d, dtype=dtype, device=DEV)
    vt = torch.zeros_like(kt)
    sk = sv = None
    R = rat.rat_cache_rows(make_cfg(B, 1, H, d, dtype, dil, win, recur, grid=grid), cap)
    ck = torch.zeros(B, H, R, d, dtype=dtype, device=DEV)
    cv = torch.zeros_like(ck)
    outs, lses = [], []
    t0 = 0
    for Tc in chunks:
        cfg = make_cfg(B, Tc, H, d, dtype, dil, win, recur, grid=grid, t0=t0, t_cap=cap)
        sl = np.s_[:, t0:t0 + Tc]
        o = torch.empty(B, Tc, H, d, dtype=dtype, device=DEV)
        lse = torch.empty(B, H, Tc, device=DEV)
        fk, fv = torch.empty(B, H, d, device=DEV), torch.empty(B, H, d, device=DEV)
        ws = rat.workspace(cfg, rat.RAT_OP_MIX_CALLER_KV)
        rat.rat_mix_prefill(cfg, q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), g[sl].contiguous(),
                            sk, sv, o, lse, kt, vt, fk, fv, ws)
        # the decode cache of the same chunk (its rows go to positions t0 + t)
        wss = rat.workspace(cfg, rat.RAT_OP_SCAN)
        rat.rat_scan_prefill(cfg, k[sl].contiguous(), v[sl].contiguous(), g[sl].contiguous(), sk, sv, None, None,
                             None, None, ck, cv, cap, wss)
        rat.rat_check_status(ws)
        rat.rat_check_status(wss)
        outs.append(o)
        lses.append(lse)
        sk, sv = fk, fv
        t0 += Tc
    rk, rfk = oracle.scan(f64(k), f64(g), None, recur)
    rv, rfv = oracle.scan(f64(v), f64(g), None, recur)
    ro, rl = oracle.attention(f64(q), rk, rv, dil, win, grid=grid)
    ft = torch.float32 if dtype == torch.float32 else dtype
    assert_close(torch.cat(outs, 1), ro, dtype, "o")
    assert_close(torch.cat(lses, 2), rl, ft, "lse")
    assert_close(kt[:, :Ttot], rk, dtype, "kt history")
    assert_close(sk, rfk, ft, "final_k")
    # every position's cache row (the layout of include/rat.h) holds the
    # oracle's augmented key and value, written chunk by chunk
    ckh, cvh = f64(ck), f64(cv)
    for h, (D, W) in enumerate(zip(dil, win)):
        S = -(-cap // D)
        for j in range(Ttot):
            if grid:
                rows = ([j // D] if j % D == D - 1 else []) + ([S + j % W] if D > 1 and W > 0 and j >= Ttot - W else [])
            else:
                rows = [(j % D) * S + j // D]
            for r in rows:
                np.testing.assert_allclose(ckh[:, h, r], rk[:, j, h], rtol=2e-2, atol=2e-2)
                np.testing.assert_allclose(cvh[:, h, r], rv[:, j, h], rtol=2e-2, atol=2e-2)


@pytest.mark.parametrize("qscale", [8, 32])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_attention_with_large_scores(dtype, qscale):
    # q scaled by 8: scores of tens in the log2 domain, so the running max
    # grows by more than the lazy-rescale threshold between tiles and P must
    # stay bounded; by 32: later tiles hold scores more than 32 above the
    # running reference, so the one-pass softmax of full tiles must raise it
    # mid-tile and rescale the P it has written; the outputs still match the
    # oracle
    B, T, H, d = 1, 4096, 2, 128
    q, kt, vt, _ = inputs(B, T, H, d, dtype, seed=91)
    q = (q.float() * qscale).to(dtype)
    dil, win = [16, 1], [256, 0]
    cfg = make_cfg(B, T, H, d, dtype, dil, win)
    o = torch.empty_like(q)
    lse = torch.empty(B, H, T, device=DEV)
    ws = rat.workspace(cfg, rat.RAT_OP_ATTN)
    rat.rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse, ws)
    rat.rat_check_status(ws)
    ro, rl = oracle.attention(f64(q), f64(kt), f64(vt), dil, win)
    assert_close(o, ro, dtype, "o")
    assert_close(lse, rl, dtype if dtype == torch.bfloat16 else torch.float32, "lse")


def test_decode_bad_position_is_reported():
    B, H, d = 2, 2, 64
    cfg = make_cfg(B, 1, H, d, torch.bfloat16, [2, 2], [0, 0])
    cap = 16
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.zeros(B, H, R, d, dtype=torch.bfloat16, device=DEV)
    cv = torch.zeros_like(ck)
    x = torch.zeros(B, H, d, dtype=torch.bfloat16, device=DEV)
    s = torch.zeros(B, H, d, device=DEV)
    ws = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
    pos = torch.tensor([3, cap], dtype=torch.int32, device=DEV)   # second entry out of range
    o = torch.empty_like(x)
    rat.rat_decode_step(cfg, x, x, x, x, s, s.clone(), ck, cv, cap, pos, o, None, ws)
    with pytest.raises(rat.RatError) as ei:
        rat.rat_check_status(ws)
    assert ei.value.status == rat.RAT_ERR_INVALID
    rat.rat_check_status(ws)  # cleared


def test_scan_lookback_timeout_is_reported_and_recovers():
    # one chunk never publishes its carry: its successors give up after the
    # bounded wait, record RAT_ERR_TIMEOUT, and the workspace stays usable
    B, T, H, d = 1, 4096, 2, 128
    dtype = torch.bfloat16
    q, k, v, g = inputs(B, T, H, d, dtype, seed=3)
    cfg = make_cfg(B, T, H, d, dtype, [1, 1], [0, 0])
    kt, vt = torch.empty_like(k), torch.empty_like(v)
    ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
    rat.rat_debug_set_scan_stall(ws, ticket=5, spin_limit_ns=20_000_000)
    rat.rat_scan_prefill(cfg, k, v, g, kt=kt, vt=vt, ws=ws)
    with pytest.raises(rat.RatError) as ei:
        rat.rat_check_status(ws)
    assert ei.value.status == rat.RAT_ERR_TIMEOUT
    rat.rat_debug_set_scan_stall(ws, ticket=-1)
    rat.rat_scan_prefill(cfg, k, v, g, kt=kt, vt=vt, ws=ws)
    rat.rat_check_status(ws)
    rk, _ = oracle.scan(f64(k), f64(g))
    assert_close(kt, rk, dtype, "kt after recovery")


# ------------------------------------------------------ full-size workloads


def worst_row_error(got, ref):
    """Largest relative L2 error of one row (last axis) of got against ref."""
    got, ref = f64(got) if isinstance(got, torch.Tensor) else got, ref
    e = np.linalg.norm(got - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
    return float(e.max())


def large_prefill_check(w, heads, n_random=24, seed=0):
    """Run the whole operator at the workload's full size on the GPU; compare
    sampled heads and rows with the oracle (which runs on those heads only).
    Besides the pooled bar, every sampled output row and EVERY row of the
    augmented keys/values of the sampled heads (all scan chunks, with their
    boundaries and carries) must be within 5e-2 on its own."""
    dtype = w.torch_dtype
    q, k, v, g = wl.prefill_inputs(w.B, w.T, w.H, w.d, w.gate_mean, dtype, device=DEV, seed=seed)
    cfg = make_cfg(w.B, w.T, w.H, w.d, dtype, w.dil, w.win, w.recur)
    out = rat.mix_prefill(cfg, q, k, v, g, want_kv=True)
    rat.rat_check_status(out["ws"])
    sl = lambda x: x[:, :, heads]
    dil = [w.dil[h] for h in heads]
    win = [w.win[h] for h in heads]
    recur = [w.recur[h] for h in heads]
    kt, fk = oracle.scan(f64(sl(k)), f64(sl(g)), None, recur)
    vt, fv = oracle.scan(f64(sl(v)), f64(sl(g)), None, recur)
    qh = f64(sl(q))
    rows = []
    for b in range(w.B):
        for i, h in enumerate(heads):
            for t in sample_rows(w.T, dil[i], win[i], n_random=n_random, seed=seed + h):
                rows.append((b, i, t))
    rows = np.array(rows)
    ro, rl = oracle.attn_rows(qh, kt, vt, dil, win, rows, parts=3)
    hsel = torch.tensor([heads[i] for i in rows[:, 1]])
    got_o = out["o"][rows[:, 0], rows[:, 2], hsel]
    got_l = out["lse"][rows[:, 0], hsel, rows[:, 2]]
    assert_close(got_o, ro, dtype, "o rows")
    assert_close(got_l, rl, dtype, "lse rows")
    e = worst_row_error(got_o, ro)
    assert e < 5e-2, "worst sampled output row: rel err %.3g" % e
    assert_close(out["final_k"][:, heads], fk, dtype, "final_k")
    assert_close(out["final_v"][:, heads], fv, dtype, "final_v")
    for name, ref in (("kt", kt), ("vt", vt)):
        got = f64(sl(out[name]))
        assert_close(got, ref, dtype, name + " (all rows of the sampled heads)")
        e = worst_row_error(got, ref)
        assert e < 5e-2, "worst %s row: rel err %.3g" % (name, e)
        del got
    del out, q, k, v, g
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_full_prefill_16k():
    large_prefill_check(wl.PREFILL_16K, heads=[0, 7, 15])


@pytest.mark.slow
def test_full_prefill_262k_window():
    large_prefill_check(wl.PREFILL_262K, heads=[0, 9], n_random=16)


@pytest.mark.slow
def test_full_prefill_262k_ragged():
    # T = 262121: D = 64 does not divide it (residues 0..40 have one row more),
    # so the dilated part runs as two classes of strided views at full size
    w = dataclasses.replace(wl.PREFILL_262K, T=wl.PREFILL_262K.T - 23)
    large_prefill_check(w, heads=[0, 9], n_random=16, seed=5)


@pytest.mark.slow
def test_full_prefill_hybrid():
    large_prefill_check(wl.HYBRID, heads=[0, 3, 4, 31], n_random=12)


@pytest.mark.slow
def test_full_decode_batch256_ctx4096():
    # the decode workload at its full batch and head count, context 4096
    w = wl.DECODE_D16
    run_decode_case(B=w.decode_batch, T=4096, steps=3, H=w.H, d=w.d, dtype=torch.bfloat16, dil=w.dil, win=w.win,
                    recur=w.recur, mu=w.gate_mean, seed=0, check_b=[0, 97, 255], check_h=[0, 5, 15],
                    gen_device=DEV)


@pytest.mark.slow
def test_hybrid_decode_full_context():
    # the hybrid workload's decode at its full 65536-token context (batch 8 of
    # the 128: the batch entries are independent)
    w = wl.HYBRID
    run_decode_case(B=8, T=65536, steps=2, H=w.H, d=w.d, dtype=torch.bfloat16, dil=w.dil, win=w.win,
                    recur=w.recur, mu=w.gate_mean, seed=0, check_b=[0, 7], check_h=[0, 3, 4, 31],
                    gen_device=DEV)

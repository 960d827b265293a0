"""Run one entry point of librat.so on a seeded synthetic case, N times.

A driver for profilers (ncu) and quick timing: it launches exactly the calls a
user would make, on inputs drawn like the operator study's workloads
(q, k, v ~ N(0,1), gate logits ~ N(mu,1)).

  python -m recurrence_augmented_dilated_gated_b200.kernel_case --op scan --T 65536
  python -m recurrence_augmented_dilated_gated_b200.kernel_case --op attn --T 65536 --dil 64 --win 512
  python -m recurrence_augmented_dilated_gated_b200.kernel_case --op decode --B 256 --ctx 4096 --dil 16
  python -m recurrence_augmented_dilated_gated_b200.kernel_case --op decode --B 256 --ctx 4096 --dil 16 --grid
  python -m recurrence_augmented_dilated_gated_b200.kernel_case --op topk --B 256 --ctx 32768 --block 64 --topk 16

--grid, --dedupe and --sep set the fixed-grid, dedupe and separate-gate flags;
--page-rows N runs the decode over a paged cache of N-row pages.
"""
import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402
import recurrence_augmented_dilated_gated_b200 as rat  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["scan", "attn", "mix", "decode", "topk"], required=True)
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--T", type=int, default=65536)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--dil", type=int, default=64)
    ap.add_argument("--win", type=int, default=0)
    ap.add_argument("--ctx", type=int, default=4096, help="decode: prefilled context")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--mu", type=float, default=2.0)
    ap.add_argument("--grid", action="store_true")
    ap.add_argument("--dedupe", action="store_true")
    ap.add_argument("--sep", action="store_true")
    ap.add_argument("--page-rows", type=int, default=0)
    ap.add_argument("--block", type=int, default=64, help="topk: block size")
    ap.add_argument("--topk", type=int, default=16, help="topk: selected blocks")
    ap.add_argument("--mode", type=int, default=0, help="topk: 0 Quest, 1 MoBA")
    a = ap.parse_args()
    dev = "cuda"
    dtype = torch.bfloat16
    H, d = a.H, a.d
    flags = ((rat.RAT_FLAG_GRID_DILATION if a.grid else 0) | (rat.RAT_FLAG_DEDUPE if a.dedupe else 0) |
             (rat.RAT_FLAG_SEPARATE_GATES if a.sep else 0))

    def gates(g):
        return torch.stack([g, g]).contiguous() if a.sep else g

    if a.op == "topk":
        T = a.ctx
        cap = T + a.iters
        cfg = rat.Config(a.B, T, H, d, dtype, [1] * H, [0] * H, flags=flags)
        q, k, v, g = wl.prefill_inputs(a.B, T, H, d, a.mu, dtype, device=dev)
        R = rat.rat_cache_rows(cfg, cap)
        ck = torch.empty(a.B, H, R, d, dtype=dtype, device=dev)
        cv = torch.empty_like(ck)
        sk = torch.empty(a.B, H, d, device=dev)
        sv = torch.empty_like(sk)
        rat.rat_scan_prefill(cfg, k, v, gates(g), None, None, None, None, sk, sv, ck, cv, cap,
                             rat.workspace(cfg, rat.RAT_OP_SCAN))
        del q, k, v, g
        stats = torch.empty(rat.topk_stats_shape(cfg, a.block, cap), device=dev)
        rat.rat_topk_build_stats(cfg, a.block, a.mode, ck, cap, stats)
        wsd = rat.workspace(cfg, rat.RAT_OP_TOPK_DECODE, cap)
        o = torch.empty(a.B, H, d, dtype=dtype, device=dev)
        for i in range(a.iters):
            tq, tk, tv, tg = wl.token_inputs(a.B, H, d, a.mu, dtype, device=dev, seed=i)
            pos = torch.full((a.B,), T + i, dtype=torch.int32, device=dev)
            rat.rat_topk_decode_step(cfg, a.block, a.topk, a.mode, tq, tk, tv, gates(tg), sk, sv, ck, cv, cap, stats,
                                     pos, o, None, None, wsd)
        rat.rat_check_status(wsd)
        return
    if a.op == "decode":
        T = a.ctx
        cap = T + a.iters
        cfg = rat.Config(a.B, T, H, d, dtype, [a.dil] * H, [a.win] * H, flags=flags)
        q, k, v, g = wl.prefill_inputs(a.B, T, H, d, a.mu, dtype, device=dev)
        R = rat.rat_cache_rows(cfg, cap)
        sk = torch.empty(a.B, H, d, device=dev)
        sv = torch.empty_like(sk)
        ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
        if a.page_rows > 0:
            # pages handed out in reverse order, so consecutive rows of a sequence are not adjacent
            pps = -(-R // a.page_rows)
            table = torch.arange(a.B * pps - 1, -1, -1, dtype=torch.int32, device=dev).view(a.B, pps)
            pool_k = torch.empty(a.B * pps, H, a.page_rows, d, dtype=dtype, device=dev)
            pool_v = torch.empty_like(pool_k)
            cache = rat.paged_cache(cfg, pool_k, pool_v, table, cap)
            rat.rat_scan_prefill_paged(cfg, k, v, gates(g), None, None, None, None, sk, sv, cache=cache,
                                       cache_cap=cap, ws=ws)
        else:
            ck = torch.empty(a.B, H, R, d, dtype=dtype, device=dev)
            cv = torch.empty_like(ck)
            rat.rat_scan_prefill(cfg, k, v, gates(g), None, None, None, None, sk, sv, ck, cv, cap, ws)
        del q, k, v, g
        wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
        o = torch.empty(a.B, H, d, dtype=dtype, device=dev)
        for i in range(a.iters):
            tq, tk, tv, tg = wl.token_inputs(a.B, H, d, a.mu, dtype, device=dev, seed=i)
            pos = torch.full((a.B,), T + i, dtype=torch.int32, device=dev)
            if a.page_rows > 0:
                rat.rat_decode_step_paged(cfg, tq, tk, tv, gates(tg), sk, sv, cache, cap, pos, o, None, wsd)
            else:
                rat.rat_decode_step(cfg, tq, tk, tv, gates(tg), sk, sv, ck, cv, cap, pos, o, None, wsd)
        rat.rat_check_status(wsd)
        return
    cfg = rat.Config(a.B, a.T, H, d, dtype, [a.dil] * H, [a.win] * H, flags=flags)
    q, k, v, g = wl.prefill_inputs(a.B, a.T, H, d, a.mu, dtype, device=dev)
    g = gates(g)
    kt, vt, o = torch.empty_like(k), torch.empty_like(v), torch.empty_like(q)
    lse = torch.empty(a.B, H, a.T, device=dev)
    op = {"scan": rat.RAT_OP_SCAN, "attn": rat.RAT_OP_ATTN, "mix": rat.RAT_OP_MIX_CALLER_KV}[a.op]
    ws = rat.workspace(cfg, op)
    for _ in range(a.iters):
        if a.op == "scan":
            rat.rat_scan_prefill(cfg, k, v, g, None, None, kt, vt, None, None, ws=ws)
        elif a.op == "attn":
            rat.rat_dilated_attn_prefill(cfg, q, k, v, o, lse, ws)
        else:
            rat.rat_mix_prefill(cfg, q, k, v, g, None, None, o, lse, kt, vt, None, None, ws)
    rat.rat_check_status(ws)


if __name__ == "__main__":
    main()

"""Run one entry point of librat.so on a seeded synthetic case, N times.

A driver for profilers (ncu) and quick timing: it launches exactly the calls a
user would make, on inputs drawn like the operator study's workloads
(q, k, v ~ N(0,1), gate logits ~ N(mu,1)).

  python -m recurrence_augmented_dilated_gated_b200.kernel_case --op scan --T 65536
  python -m recurrence_augmented_dilated_gated_b200.kernel_case --op attn --T 65536 --dil 64 --win 512
  python -m recurrence_augmented_dilated_gated_b200.kernel_case --op decode --B 256 --ctx 4096 --dil 16
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
    ap.add_argument("--op", choices=["scan", "attn", "mix", "decode"], required=True)
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--T", type=int, default=65536)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--dil", type=int, default=64)
    ap.add_argument("--win", type=int, default=0)
    ap.add_argument("--ctx", type=int, default=4096, help="decode: prefilled context")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--mu", type=float, default=2.0)
    a = ap.parse_args()
    dev = "cuda"
    dtype = torch.bfloat16
    H, d = a.H, a.d
    if a.op == "decode":
        T = a.ctx
        cap = T + a.iters
        cfg = rat.Config(a.B, T, H, d, dtype, [a.dil] * H, [a.win] * H)
        q, k, v, g = wl.prefill_inputs(a.B, T, H, d, a.mu, dtype, device=dev)
        R = rat.rat_cache_rows(cfg, cap)
        ck = torch.empty(a.B, H, R, d, dtype=dtype, device=dev)
        cv = torch.empty_like(ck)
        sk = torch.empty(a.B, H, d, device=dev)
        sv = torch.empty_like(sk)
        ws = rat.workspace(cfg, rat.RAT_OP_SCAN)
        rat.rat_scan_prefill(cfg, k, v, g, None, None, None, None, sk, sv, ck, cv, cap, ws)
        del q, k, v, g
        wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap)
        o = torch.empty(a.B, H, d, dtype=dtype, device=dev)
        for i in range(a.iters):
            tq, tk, tv, tg = wl.token_inputs(a.B, H, d, a.mu, dtype, device=dev, seed=i)
            pos = torch.full((a.B,), T + i, dtype=torch.int32, device=dev)
            rat.rat_decode_step(cfg, tq, tk, tv, tg, sk, sv, ck, cv, cap, pos, o, None, wsd)
        rat.rat_check_status(wsd)
        return
    cfg = rat.Config(a.B, a.T, H, d, dtype, [a.dil] * H, [a.win] * H)
    q, k, v, g = wl.prefill_inputs(a.B, a.T, H, d, a.mu, dtype, device=dev)
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

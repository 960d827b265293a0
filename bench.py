#!/usr/bin/env python
"""Benchmark of the RAT+ temporal-mixing operator on B200.

Headline workload: prefill of 262144 tokens, B=1, 16 heads x 128 (hidden
2048), dilation 64 plus a local window of 512 merged by log-sum-exp, bf16
operands with fp32 state and softmax (the 262K prefill of "RAT+: Train Dense,
Infer Sparse", Figure 2).  One step = one pass of the whole operator over that
input: the recurrence scan of k and v, then the dilated + windowed attention.
Alongside: decode at batch 256, 16 heads x 128, D=16 over a prefilled cache
(Figure 2's decode scenario), reported in the "decode" object.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronize; CUDA events on the launching stream time the whole step
and each kernel stage; the multi-GPU time is the max over ranks.  Inputs are
larger than L2 (4.3 GB per prefill step), so no flush is needed.

`--impl reference` times the CPU oracle (the plain fp64 implementation the
parity tests use) on the host cores on a bounded sample of the same workload.

Prints ONE JSON line on rank 0.
"""
import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "temporal-mix prefill tok/s @262K & decode tok/s; % of HBM/tensor roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
RAGGED_T = 262144 - 23   # a long prefill whose length the dilation does not divide
NOMINAL_HBM_GBS = 8000.0   # the ~8 TB/s nominal HBM3e figure, reported beside the measured copy peak


# ----------------------------------------------------------------- plumbing


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(world, backend):
    import torch.distributed as dist
    from datetime import timedelta

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return dist


def max_over_ranks(x, world, device):
    """Max of a float over ranks (identity at world size 1)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["_source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["_source"] = "fallback"
    return d


class NvmlSampler:
    """SM clock and throttle reasons read through NVML every ~5 ms on a host
    thread, with host timestamps, so that even a short timed region holds
    several samples.  The GPU is found by its PCI bus id (CUDA and NVML
    number devices differently when CUDA_VISIBLE_DEVICES is set)."""

    PERIOD_S = 0.005

    def __init__(self, cuda_index):
        import threading

        import pynvml

        self.nv = pynvml
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(cuda_index)
        bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        bits = {"hw_slowdown": "HwSlowdown", "hw_thermal_slowdown": "HwThermalSlowdown",
                "sw_thermal_slowdown": "SwThermalSlowdown", "sw_power_cap": "SwPowerCap"}
        self.bits = {k: getattr(pynvml, "nvmlClocksEventReason" + v, None) or
                     getattr(pynvml, "nvmlClocksThrottleReason" + v) for k, v in bits.items()}
        self.reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        self.samples = []
        self._stop = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            t = time.time()
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = int(self.reasons_fn(self.h))
            except nv.NVMLError:
                break
            self.samples.append((t, sm, self.max_mhz, {k for k, b in self.bits.items() if r & b}))
            self._stop.wait(self.PERIOD_S)

    def start(self):
        self.thread.start()
        return self

    def stop(self):
        self._stop.set()
        self.thread.join(timeout=5)


class ClockSampler:
    """SM clocks and throttle reasons during the run: NVML every ~5 ms, or
    nvidia-smi every 100 ms where NVML cannot be used; host timestamps let
    summary() pick the samples inside the timed region."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.f = None
        self.nvml = None

    def start(self):
        try:
            self.nvml = NvmlSampler(self.gpu).start()
            return self
        except Exception:  # no NVML here: fall back to nvidia-smi
            self.nvml = None
        try:
            self.f = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        return self

    def stop(self):
        if self.nvml is not None:
            self.nvml.stop()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        """Median SM clock and active throttle reasons of the samples taken in
        [t0, t1] (host epoch seconds); all samples when fewer than 2 fall there."""
        import datetime

        samples = []
        source = "nvidia-smi, 100 ms"
        if self.nvml is not None:
            samples, source = list(self.nvml.samples), "nvml, 5 ms"
        elif self.proc is None or self.f is None:
            return None
        else:
            self.f.seek(0)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in ([] if self.nvml is not None else self.f.read().strip().splitlines()):
            r = [x.strip() for x in line.split(",")]
            if len(r) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx = float(r[2]), float(r[3])
            except ValueError:
                continue
            active = {n for i, n in enumerate(names) if r[6 + i].lower().startswith("active")}
            samples.append((ts, sm, mx, active))
        if not samples:
            return None
        window = "timed region"
        sel = [x for x in samples if t0 is not None and t0 - 0.05 <= x[0] <= t1 + 0.05]
        if len(sel) < 2:
            sel, window = samples, "warm-up + timed region (timed region shorter than the sampling interval)"
        reasons = set()
        for x in sel:
            reasons |= x[3]
        return {"sm_mhz": float(np.median([x[1] for x in sel])), "sm_max_mhz": float(max(x[2] for x in sel)),
                "samples": len(sel), "reasons": sorted(reasons), "window": window, "source": source}


def profile_traffic(name, key=None):
    """Per-launch DRAM bytes from the committed ncu summary profiles/<name>.md
    (line `traffic_bytes_per_launch[key]: ...` when key is given), or None if
    there is none or the kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", name + ".md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    tag = r"\[" + re.escape(key) + r"\]" if key else ""
    m = re.search(r"traffic_bytes_per_launch" + tag + r":\s*([0-9.eE+]+)\s*\(source sha1 ([0-9a-f]+) of ([\w./]+)\)", txt)
    if not m:
        return None
    src = os.path.join(ROOT, m.group(3))
    if not os.path.exists(src) or hashlib.sha1(open(src, "rb").read()).hexdigest()[:12] != m.group(2)[:12]:
        return None
    return float(m.group(1))


# --------------------------------------------------------- algorithmic work


def attn_pairs(T, D, W):
    """Unmasked (query, key) pairs of one head: dilated part + window part."""
    n = np.array([(T - r + D - 1) // D for r in range(min(D, T))], dtype=np.float64)
    pairs = float(np.sum(n * (n + 1) / 2))
    if W > 0:
        Wm = min(W, T)
        pairs += Wm * (Wm + 1) / 2 + (T - Wm) * W
    return pairs


def variant_pairs(T, D, W, grid=False, dedupe=False, t_from=0):
    """Unmasked (query, key) pairs of one head's rows t_from .. T-1 under the
    fixed-grid reading (keys j <= t with j mod D == D-1, plus t once) and/or
    dedupe (the window part skips the dilated set's keys), in closed form per row."""
    t = np.arange(t_from, T, dtype=np.int64)
    lo = np.maximum(0, t - W + 1)
    if grid:
        on = (t % D) == D - 1
        n_dil = (t + 1) // D + np.where(on, 0, 1)
    else:
        n_dil = t // D + 1
    n_win = np.minimum(W, t + 1) if W > 0 else np.zeros_like(t)
    if dedupe and W > 0:
        if grid:    # grid positions in [lo, t], plus t itself when it is off the grid
            shared = (t + 1) // D - lo // D + np.where(on, 0, 1)
        else:       # t, t-D, ... down to lo
            shared = (t - lo) // D + 1
        n_win = n_win - shared
    return float(np.sum(n_dil + n_win))


def prefill_work(w):
    """(attention FLOPs, scan bytes) of one prefill step: 4*d FLOPs per pair;
    10 bytes per (token, channel) of a recurrent head (k, v, g read; kt, vt written)."""
    flops = 0.0
    scan_bytes = 0.0
    elt = 2 if w.dtype == "bf16" else 4
    for h in range(w.H):
        flops += w.B * 4.0 * w.d * attn_pairs(w.T, w.dil[h], w.win[h])
        if w.recur[h]:
            scan_bytes += w.B * w.T * w.d * 5 * elt
    return flops, scan_bytes


def decode_bytes(B, H, d, t, dil, win, elt=2):
    """Algorithmic HBM bytes of one decode step at position t: every attended
    cache row read once (K~ and V~), plus the token's q,k,v,g, o, the fp32 state
    read+write and the new cache row."""
    rows = 0
    for h in range(H):
        rows += t // dil[h] + (min(win[h], t + 1) - 1 if win[h] > 0 else 0)
    return B * (rows * 2 * d * elt + H * d * (5 * elt + 16 + 2 * elt))


# --------------------------------------------------------------- prefill


def bench_prefill(rat, w, steps, warmup, world, rank, dev, e2e_steps, mix=False):
    """Time `steps` prefill steps of workload w.  By default a step is
    rat_scan_prefill then rat_dilated_attn_prefill (= rat_mix_prefill with
    caller K~/V~), with events around each stage.  mix=True times
    rat_mix_prefill itself with K~/V~ kept in its workspace, as a user calls
    it (heads without recurrence then attend to k/v without a copy), and the
    attention stage alone in a second timed loop."""
    if mix:
        return bench_prefill_mix(rat, w, steps, warmup, world, rank, dev)
    dtype = w.torch_dtype
    q, k, v, g = wl.prefill_inputs(w.B, w.T, w.H, w.d, w.gate_mean, dtype, device=dev, seed=rank)
    cfg = rat.Config(w.B, w.T, w.H, w.d, dtype, w.dil, w.win, w.recur)
    kt, vt = torch.empty_like(k), torch.empty_like(v)
    o = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32, device=dev)
    fk = torch.empty(w.B, w.H, w.d, dtype=torch.float32, device=dev)
    fv = torch.empty_like(fk)
    ws = rat.workspace(cfg, rat.RAT_OP_MIX_CALLER_KV, device=dev)
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        rat.rat_scan_prefill(cfg, k, v, g, None, None, kt, vt, fk, fv, ws=ws, stream=stream)
        if evs:
            evs[1].record(stream)
        rat.rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse, ws=ws, stream=stream)
        if evs:
            evs[2].record(stream)

    clk = ClockSampler(torch.cuda.current_device()).start()
    for _ in range(warmup):
        step()
    rat.rat_check_status(ws)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    n0 = rat.rat_launch_count()
    t_host0 = time.time()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    t_host1 = time.time()
    clk.stop()
    launches = rat.rat_launch_count() - n0
    barrier(world)
    rat.rat_check_status(ws)
    scan_ms = [e[0].elapsed_time(e[1]) for e in evs]
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = evs[0][0].elapsed_time(evs[-1][2])
    total_ms = max_over_ranks(total_ms, world, dev)
    res = dict(total_ms=total_ms, scan_ms=float(np.mean(scan_ms)), attn_ms=float(np.mean(attn_ms)),
               launches=launches, clocks=clk.summary(t_host0, t_host1))

    # End to end through the user call with host buffers: every step copies
    # its q, k, v, g in from pinned memory, runs rat_mix_prefill and copies o
    # back out.  As in a serving loop, the steps are pipelined on three
    # streams with double-buffered device tensors: the copy-in of step i+1 and
    # the copy-out of step i-1 overlap the compute of step i (PCIe is full
    # duplex).  Events order every buffer's reuse.
    if e2e_steps > 0:
        hq, hk, hv, hg = (x.cpu().pin_memory() for x in (q, k, v, g))
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        wsm = rat.workspace(cfg, rat.RAT_OP_MIX, device=dev)
        del kt, vt
        torch.cuda.empty_cache()
        ins = [(q, k, v, g), tuple(torch.empty_like(x) for x in (q, k, v, g))]
        outs = [o, torch.empty_like(o)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        in_ready = [ev(), ev()]      # copy-in of the slot done
        comp_done = [ev(), ev()]     # compute of the slot done (inputs free, output ready)
        out_done = [ev(), ev()]      # copy-out of the slot done (output free)

        def run(nsteps, t0=None, t1=None):
            for i in range(nsteps + 2):
                if i < nsteps:           # copy-in of step i
                    sl = i % 2
                    with torch.cuda.stream(s_in):
                        if i >= 2:
                            s_in.wait_event(comp_done[sl])
                        if i == 0 and t0 is not None:
                            t0.record(s_in)
                        for d_, h_ in zip(ins[sl], (hq, hk, hv, hg)):
                            d_.copy_(h_, non_blocking=True)
                        in_ready[sl].record(s_in)
                j = i - 1
                if 0 <= j < nsteps:      # compute of step j
                    sl = j % 2
                    stream.wait_event(in_ready[sl])
                    if j >= 2:
                        stream.wait_event(out_done[sl])
                    qq, kk, vv, gg = ins[sl]
                    rat.rat_mix_prefill(cfg, qq, kk, vv, gg, None, None, outs[sl], None, None, None, fk, fv,
                                        ws=wsm, stream=stream)
                    comp_done[sl].record(stream)
                j = i - 2
                if 0 <= j < nsteps:      # copy-out of step j
                    sl = j % 2
                    with torch.cuda.stream(s_out):
                        s_out.wait_event(comp_done[sl])
                        ho[sl].copy_(outs[sl], non_blocking=True)
                        out_done[sl].record(s_out)
                        if j == nsteps - 1 and t1 is not None:
                            t1.record(s_out)

        run(2)
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run(e2e_steps, a, b)
        torch.cuda.synchronize()
        rat.rat_check_status(wsm)
        e_ms = max_over_ranks(a.elapsed_time(b), world, dev) / e2e_steps
        res["e2e_ms"] = e_ms
        res["h2d_bytes"] = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hg))
        res["d2h_bytes"] = ho[0].numel() * ho[0].element_size()
        del wsm, hq, hk, hv, hg, ho, ins, outs
    del q, k, v, g, o, lse, ws
    torch.cuda.empty_cache()
    return res


def bench_prefill_mix(rat, w, steps, warmup, world, rank, dev):
    dtype = w.torch_dtype
    q, k, v, g = wl.prefill_inputs(w.B, w.T, w.H, w.d, w.gate_mean, dtype, device=dev, seed=rank)
    cfg = rat.Config(w.B, w.T, w.H, w.d, dtype, w.dil, w.win, w.recur)
    o = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32, device=dev)
    fk = torch.empty(w.B, w.H, w.d, dtype=torch.float32, device=dev)
    fv = torch.empty_like(fk)
    ws = rat.workspace(cfg, rat.RAT_OP_MIX, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        barrier(world)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n0 = rat.rat_launch_count()
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), world, dev), rat.rat_launch_count() - n0

    mix = lambda: rat.rat_mix_prefill(cfg, q, k, v, g, None, None, o, lse, None, None, fk, fv, ws=ws,
                                      stream=stream)
    clk = ClockSampler(torch.cuda.current_device()).start()
    for _ in range(warmup):
        mix()
    rat.rat_check_status(ws)
    t_host0 = time.time()
    total_ms, launches = timed(mix, steps)
    t_host1 = time.time()
    clk.stop()
    rat.rat_check_status(ws)
    del ws
    torch.cuda.empty_cache()
    # the scan stage alone (rat_scan_prefill into caller K~/V~, which also
    # copies the k/v of heads without recurrence), then the attention stage
    # alone over those augmented keys/values
    kt, vt = torch.empty_like(k), torch.empty_like(v)
    wss = rat.workspace(cfg, rat.RAT_OP_SCAN, device=dev)
    scan = lambda: rat.rat_scan_prefill(cfg, k, v, g, None, None, kt, vt, fk, fv, ws=wss, stream=stream)
    for _ in range(warmup):
        scan()
    scan_total, _ = timed(scan, steps)
    rat.rat_check_status(wss)
    del wss, k, v, g
    wsa = rat.workspace(cfg, rat.RAT_OP_ATTN, device=dev)
    attn = lambda: rat.rat_dilated_attn_prefill(cfg, q, kt, vt, o, lse, ws=wsa, stream=stream)
    for _ in range(warmup):
        attn()
    attn_total, _ = timed(attn, steps)
    rat.rat_check_status(wsa)
    del q, kt, vt, o, lse, wsa
    torch.cuda.empty_cache()
    plain = sum(1 for h in range(w.H) if not w.recur[h])
    return dict(total_ms=total_ms, attn_ms=attn_total / steps, scan_ms=scan_total / steps,
                scan_copy_bytes=float(w.B * w.T * plain * w.d * 4 * (2 if w.dtype == "bf16" else 4)),
                launches=launches, clocks=clk.summary(t_host0, t_host1))


# ---------------------------------------------------------------- decode


def bench_decode(rat, w, ctx, steps, warmup, world, rank, dev, fill_chunk=8, flags=0, page_rows=0):
    """Fill the cache of `ctx` tokens with batch-chunked rat_scan_prefill, then
    time `steps` decode steps (positions ctx+warmup .. ).  flags: RAT_FLAG_*;
    page_rows > 0: the decode reads a paged copy of the cache (pages in
    reverse order, so no two consecutive pages of a sequence are adjacent)."""
    dtype = w.torch_dtype
    B = w.decode_batch
    cap = ctx + warmup + steps
    cfg = rat.Config(B, ctx, w.H, w.d, dtype, w.dil, w.win, w.recur, flags=flags)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.empty(B, w.H, R, w.d, dtype=dtype, device=dev)
    cv = torch.empty_like(ck)
    sk = torch.empty(B, w.H, w.d, dtype=torch.float32, device=dev)
    sv = torch.empty_like(sk)
    ccfg = rat.Config(fill_chunk, ctx, w.H, w.d, dtype, w.dil, w.win, w.recur, flags=flags)
    wsc = rat.workspace(ccfg, rat.RAT_OP_SCAN, device=dev)
    per_b = w.H * R * w.d
    for b0 in range(0, B, fill_chunk):
        k, v, g = wl.prefill_inputs(fill_chunk, ctx, w.H, w.d, w.gate_mean, dtype, device=dev,
                                    seed=1000 + rank * 997 + b0)[1:]
        rat.rat_scan_prefill(ccfg, k, v, g, None, None, None, None, sk[b0:b0 + fill_chunk], sv[b0:b0 + fill_chunk],
                             ck.view(-1)[b0 * per_b:(b0 + fill_chunk) * per_b],
                             cv.view(-1)[b0 * per_b:(b0 + fill_chunk) * per_b], cap, ws=wsc)
        del k, v, g
    rat.rat_check_status(wsc)
    del wsc
    cache = None
    if page_rows > 0:
        # the same logical rows moved into shuffled pages
        pps = -(-R // page_rows)
        table = torch.arange(B * pps - 1, -1, -1, dtype=torch.int32, device=dev).view(B, pps)
        pool_k = torch.zeros(B * pps, w.H, page_rows, w.d, dtype=dtype, device=dev)
        pool_v = torch.zeros_like(pool_k)
        r = torch.arange(R, device=dev)
        for b in range(B):
            pg = table[b, r // page_rows].long()
            pool_k[pg, :, r % page_rows] = ck[b].transpose(0, 1)
            pool_v[pg, :, r % page_rows] = cv[b].transpose(0, 1)
        del ck, cv
        ck = cv = None
        cache = rat.paged_cache(cfg, pool_k, pool_v, table, cap)
    n = warmup + steps
    toks = [wl.token_inputs(B, w.H, w.d, w.gate_mean, dtype, device=dev, seed=5000 + i) for i in range(n)]
    poss = [torch.full((B,), ctx + i, dtype=torch.int32, device=dev) for i in range(n)]
    o = torch.empty(B, w.H, w.d, dtype=dtype, device=dev)
    wsd = rat.workspace(cfg, rat.RAT_OP_DECODE, cap, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        tq, tk, tv, tg = toks[i]
        if cache is not None:
            rat.rat_decode_step_paged(cfg, tq, tk, tv, tg, sk, sv, cache, cap, poss[i], o, None, ws=wsd, stream=stream)
        else:
            rat.rat_decode_step(cfg, tq, tk, tv, tg, sk, sv, ck, cv, cap, poss[i], o, None, ws=wsd, stream=stream)

    for i in range(warmup):
        step(i)
    rat.rat_check_status(wsd)
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = rat.rat_launch_count()
    a.record(stream)
    for i in range(warmup, n):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    launches = rat.rat_launch_count() - n0
    rat.rat_check_status(wsd)
    ms = max_over_ranks(a.elapsed_time(b), world, dev) / steps
    t_mid = ctx + warmup + steps // 2
    byts = decode_bytes(B, w.H, w.d, t_mid, w.dil, w.win)
    del ck, cv, toks, cache
    torch.cuda.empty_cache()
    return dict(ms=ms, bytes=byts, launches=launches, ctx=ctx)


def bench_attn_variant(rat, w, flags, steps, warmup, world, rank, dev, t0=0, T=None):
    """The attention step alone (rat_dilated_attn_prefill) on the prefill
    workload under RAT_FLAG_* `flags`; with t0 > 0, only the queries of
    positions t0 .. T-1 (the last chunk of a chunked prefill) over the whole
    history; T overrides the workload's length.  Returns ms per launch."""
    dtype = w.torch_dtype
    T = T or w.T
    q, k, v, _ = wl.prefill_inputs(w.B, T, w.H, w.d, w.gate_mean, dtype, device=dev, seed=11 + rank)
    if t0 > 0:
        q = q[:, t0:].contiguous()
    cfg = rat.Config(w.B, T - t0, w.H, w.d, dtype, w.dil, w.win, w.recur, flags=flags, t0=t0)
    o = torch.empty_like(q)
    ws = rat.workspace(cfg, rat.RAT_OP_ATTN, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        rat.rat_dilated_attn_prefill(cfg, q, k, v, o, None, ws, stream=stream)
    rat.rat_check_status(ws)
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = rat.rat_launch_count()
    a.record(stream)
    for _ in range(steps):
        rat.rat_dilated_attn_prefill(cfg, q, k, v, o, None, ws, stream=stream)
    b.record(stream)
    torch.cuda.synchronize()
    launches = rat.rat_launch_count() - n0
    rat.rat_check_status(ws)
    ms = max_over_ranks(a.elapsed_time(b), world, dev) / steps
    del q, k, v, o, ws
    torch.cuda.empty_cache()
    return dict(ms=ms, launches=launches)


def topk_decode_bytes(B, H, d, t, block, K, elt=2):
    """Algorithmic HBM bytes of one top-k decode step at position t: the fp32
    statistics of the candidate blocks, the old rows (before t) of the first,
    local and selected blocks (K~ and V~), the token's q,k,v,g, o, the state,
    and the new row plus its block's statistics (the new row itself is
    attended from registers, as in decode_bytes)."""
    c = t // block
    ncand = max(0, c - 1)
    rows = t if c == 0 else block + min(K, ncand) * block + (t - c * block)
    stats = ncand * 2 * d * 4
    return B * H * (stats + rows * 2 * d * elt + d * (5 * elt + 16 + 2 * elt) + 2 * 2 * d * 4)


def bench_topk(rat, B, H, d, ctx, block, K, mode, steps, warmup, world, rank, dev, fill_chunk=8, gate_mean=2.0):
    """Top-k block decode over a dense cache of `ctx` tokens: batch-chunked
    prefill into the cache, block statistics, then `steps` timed steps."""
    dtype = torch.bfloat16
    cap = ctx + warmup + steps
    dil, win = [1] * H, [0] * H
    cfg = rat.Config(B, ctx, H, d, dtype, dil, win)
    R = rat.rat_cache_rows(cfg, cap)
    ck = torch.empty(B, H, R, d, dtype=dtype, device=dev)
    cv = torch.empty_like(ck)
    sk = torch.empty(B, H, d, device=dev)
    sv = torch.empty_like(sk)
    ccfg = rat.Config(fill_chunk, ctx, H, d, dtype, dil, win)
    wsc = rat.workspace(ccfg, rat.RAT_OP_SCAN, device=dev)
    per_b = H * R * d
    for b0 in range(0, B, fill_chunk):
        k, v, g = wl.prefill_inputs(fill_chunk, ctx, H, d, gate_mean, dtype, device=dev, seed=3000 + rank * 997 + b0)[1:]
        rat.rat_scan_prefill(ccfg, k, v, g, None, None, None, None, sk[b0:b0 + fill_chunk], sv[b0:b0 + fill_chunk],
                             ck.view(-1)[b0 * per_b:(b0 + fill_chunk) * per_b],
                             cv.view(-1)[b0 * per_b:(b0 + fill_chunk) * per_b], cap, ws=wsc)
        del k, v, g
    rat.rat_check_status(wsc)
    del wsc
    stats = torch.empty(rat.topk_stats_shape(cfg, block, cap), device=dev)
    rat.rat_topk_build_stats(cfg, block, mode, ck, cap, stats)
    n = warmup + steps
    toks = [wl.token_inputs(B, H, d, gate_mean, dtype, device=dev, seed=7000 + i) for i in range(n)]
    poss = [torch.full((B,), ctx + i, dtype=torch.int32, device=dev) for i in range(n)]
    o = torch.empty(B, H, d, dtype=dtype, device=dev)
    wsd = rat.workspace(cfg, rat.RAT_OP_TOPK_DECODE, cap, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        tq, tk, tv, tg = toks[i]
        rat.rat_topk_decode_step(cfg, block, K, mode, tq, tk, tv, tg, sk, sv, ck, cv, cap, stats, poss[i], o, None,
                                 None, ws=wsd, stream=stream)

    for i in range(warmup):
        step(i)
    rat.rat_check_status(wsd)
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = rat.rat_launch_count()
    a.record(stream)
    for i in range(warmup, n):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    launches = rat.rat_launch_count() - n0
    rat.rat_check_status(wsd)
    ms = max_over_ranks(a.elapsed_time(b), world, dev) / steps
    byts = topk_decode_bytes(B, H, d, ctx + warmup + steps // 2, block, K)
    del ck, cv, stats, toks
    torch.cuda.empty_cache()
    return dict(ms=ms, bytes=byts, launches=launches, ctx=ctx)


# ------------------------------------------------------------ CPU oracle


def oracle_sample(w, n_rows, seed=0, rows_offset=0.5):
    """Time the CPU oracle on one head of each head class of the workload (a
    class = heads with the same dilation, window and recurrence flag): the
    full-length scan of k and v, then `n_rows` query rows spread evenly over T.
    Returns the extrapolated whole-operator throughput (tokens/s over all
    heads and batch entries) and the seconds the sample took."""
    import oracle

    classes = {}
    for h in range(w.H):
        classes.setdefault((w.dil[h], w.win[h], w.recur[h]), []).append(h)
    q, k, v, g = wl.prefill_inputs(1, w.T, 1, w.d, w.gate_mean, w.torch_dtype, device="cpu", seed=seed)
    f = lambda x: x.float().numpy().astype(np.float64)
    q, k, v, g = f(q), f(k), f(v), f(g)
    ts = ((np.arange(n_rows) + rows_offset) * w.T / n_rows).astype(np.int64)
    rows = np.stack([np.zeros_like(ts), np.zeros_like(ts), ts], axis=1)
    per_seq, spent = 0.0, 0.0
    for (D, W, rec), heads in classes.items():
        t0 = time.perf_counter()
        kt, _ = oracle.scan(k, g, None, [rec])
        vt, _ = oracle.scan(v, g, None, [rec])
        t_scan = time.perf_counter() - t0
        t0 = time.perf_counter()
        oracle.attn_rows(q, kt, vt, [D], [W], rows, parts=3)
        t_rows = time.perf_counter() - t0
        per_seq += len(heads) * (t_scan + t_rows * (w.T / n_rows))
        spent += t_scan + t_rows
    tok_s = w.T / per_seq
    return tok_s, spent


def oracle_decode_sample(w, ctx, seed=0):
    """Time one oracle decode step of one batch entry (all heads) at position
    ctx over a random history; a step of the whole batch costs B times that.
    Returns (tokens/s, seconds spent)."""
    import oracle

    H, d = w.H, w.d
    rng = np.random.default_rng(seed)
    # the oracle's work does not depend on the values: a constant history
    hist_k = np.full((1, ctx + 1, H, d), 0.25)
    hist_v = np.full((1, ctx + 1, H, d), 0.5)
    sk, sv = rng.standard_normal((1, H, d)), rng.standard_normal((1, H, d))
    q, k, v = (rng.standard_normal((1, H, d)) for _ in range(3))
    g = rng.standard_normal((1, H, d)) + w.gate_mean
    n, t0 = 0, time.perf_counter()
    while True:   # repeat the step (same position) for at least 0.2 s
        oracle.decode_step(q, k, v, g, sk, sv, hist_k, hist_v, [ctx], w.dil, w.win, w.recur)
        n += 1
        sec = time.perf_counter() - t0
        if sec >= 0.2:
            break
    return n / sec, sec


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle as it stands, rank 0 only."""
    if rank != 0:
        return
    w = wl.PREFILL_262K
    n_rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(w, max(16, n_rows // 8))
    vals, secs = [], []
    for i in range(args.steps):
        v, s = oracle_sample(w, n_rows, rows_offset=(i % 4 + 0.5) / 4)
        vals.append(v)
        secs.append(s)
    value = float(np.mean(vals))
    cores = host_cores()
    sample = ("head 0 of %d: full scan of k and v over T=%d plus %d query rows spread over T per step; "
              "extrapolated to all heads" % (w.H, w.T, n_rows))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean(secs)) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "global_batch": w.B, "seq_len": w.T, "parallelism": "host threads"},
            "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main


def hbm_roofline(byts, ms, peaks, traffic=None):
    gbs = byts / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"], "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS, "traffic": traffic,
            "peak_source": peaks["_source"] + " copy"}


def tensor_roofline(flops, ms, peaks, traffic=None, kernel=None):
    tf = flops / (ms * 1e-3) / 1e12
    r = {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
         "frac": tf / peaks["bf16_tflops"], "traffic": traffic, "peak_source": peaks["_source"] + " bf16 dense burst"}
    if kernel:
        r = dict(kernel=kernel, **r)
    return r


def prefill_entry(w, r, steps, world, peaks, cpu=None):
    """One prefill workload's line: whole-step tok/s, the attention stage
    against the bf16 tensor peak and the scan stage against HBM."""
    flops, scan_bytes = prefill_work(w)
    scan_bytes += r.get("scan_copy_bytes", 0.0)
    step_ms = r["total_ms"] / steps
    e = {"workload": w.name, "value": w.B * w.T * world / (step_ms * 1e-3), "unit": "tok/s",
         "ms_per_step": step_ms, "kernels_ms": {"scan": r["scan_ms"], "attention": r["attn_ms"]},
         "roofline": tensor_roofline(flops, r["attn_ms"], peaks, kernel="attention"),
         "scan_roofline": hbm_roofline(scan_bytes, r["scan_ms"], peaks) if r["scan_ms"] > 0 else None,
         "gpu_launches": r["launches"], "clocks": r["clocks"]}
    if "scan_copy_bytes" in r:
        e["step"] = ("rat_mix_prefill (K~/V~ in its workspace, heads without recurrence read k/v directly); "
                     "the scan (into caller K~/V~, copying those heads' k/v: 4 B per token-channel each way) "
                     "and the attention timed alone")
    if cpu:
        e["cpu_baseline"] = cpu
    return e


def decode_entry(w, r, steps, world, peaks, traffic=None, cpu=None):
    e = {"ctx": r["ctx"], "value": w.decode_batch * world / (r["ms"] * 1e-3), "unit": "tok/s",
         "ms_per_step": r["ms"], "steps": steps, "roofline": hbm_roofline(r["bytes"], r["ms"], peaks, traffic),
         "gpu_launches": r["launches"]}
    if cpu:
        e["cpu_baseline"] = cpu
    return e


def cpu_entry(v, secs, what):
    return {"value": v, "unit": "tok/s", "cores": host_cores(), "kind": "oracle", "sample": "%s (%.1f s)" % (what, secs)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-ctx", type=str, default="4096,16384,32768")
    ap.add_argument("--decode-steps", type=int, default=0,
                    help="decode steps per context (0: the workload's own horizon, 1024 and 256)")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-rows", type=int, default=2048, help="oracle rows timed for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=512, help="oracle rows per reference-arm step")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (16K prefill, hybrid prefill and decode)")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the decode variants (fixed grid, paged cache, top-k blocks)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_env()
    if args.impl == "reference":
        init_dist(world, "gloo")
        run_reference(args, world, rank)
        return

    import recurrence_augmented_dilated_gated_b200 as rat

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    rat.load_library()
    peaks = load_peaks()
    cpu_ok = not args.no_cpu and world == 1

    w = wl.PREFILL_262K
    pre = bench_prefill(rat, w, args.steps, args.warmup, world, rank, dev, args.e2e_steps)
    flops, scan_bytes = prefill_work(w)
    tokens = w.B * w.T * world
    step_ms = pre["total_ms"] / args.steps
    value = tokens / (step_ms * 1e-3)

    wd = wl.DECODE_D16
    dsteps = args.decode_steps or wd.decode_steps
    dec = []
    for ctx in [int(c) for c in args.decode_ctx.split(",") if c]:
        dec.append(bench_decode(rat, wd, ctx, dsteps, args.warmup, world, rank, dev))

    cfgs = {}
    if not args.no_configs:
        w2, w5 = wl.PREFILL_16K, wl.HYBRID
        cfgs["prefill_16k"] = (w2, bench_prefill(rat, w2, args.steps, args.warmup, world, rank, dev, 0))
        cfgs["prefill_hybrid"] = (w5, bench_prefill(rat, w5, args.steps, args.warmup, world, rank, dev, 0, mix=True))
        h_steps = args.decode_steps or w5.decode_steps
        cfgs["decode_hybrid"] = (w5, bench_decode(rat, w5, w5.decode_ctx[0], h_steps, args.warmup, world, rank, dev,
                                                  fill_chunk=4), h_steps)

    nxt = {}
    if not args.no_next_rows:
        vsteps = min(dsteps, 64)
        nxt["grid_decode"] = bench_decode(rat, wd, 4096, vsteps, args.warmup, world, rank, dev,
                                          flags=rat.RAT_FLAG_GRID_DILATION)
        nxt["paged_decode"] = bench_decode(rat, wd, 4096, vsteps, args.warmup, world, rank, dev, page_rows=256)
        att_var = {name: bench_attn_variant(rat, w, f, 3, args.warmup, world, rank, dev)
                   for name, f in (("grid", rat.RAT_FLAG_GRID_DILATION), ("dedupe", rat.RAT_FLAG_DEDUPE))}
        att_var["chunked"] = bench_attn_variant(rat, w, 0, 3, args.warmup, world, rank, dev, t0=w.T * 3 // 4)
        att_var["ragged"] = bench_attn_variant(rat, w, 0, 3, args.warmup, world, rank, dev, T=RAGGED_T)
        nxt["topk_decode"] = bench_topk(rat, wd.decode_batch, wd.H, wd.d, 16384, 64, 16, rat.RAT_TOPK_QUEST,
                                        vsteps, args.warmup, world, rank, dev)

    if rank != 0:
        return
    attn_tflops = flops / (pre["attn_ms"] * 1e-3) / 1e12
    scan_gbs = scan_bytes / (pre["scan_ms"] * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tok/s",
        "value_is": "prefill tokens/s of the whole operator (scan + dilated/window attention) at T=262144",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (q,k,v ~ N(0,1), gate logits ~ N(2,1), seeded)",
        "config": {"workload": w.name, "global_batch": w.B * world, "seq_len": w.T,
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (4.3 GB per step), no flush"},
        "roofline": {"bound": "tensor", "kernel": "attention (dilated + window + LSE merge)",
                     "achieved": attn_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": attn_tflops / peaks["bf16_tflops"],
                     "traffic": profile_traffic("attn_prefill262k"),
                     "algorithmic": "%.4g FLOP per launch (4*d per unmasked pair)" % flops,
                     "peak_source": peaks["_source"] + " bf16 dense burst"},
        "scan_roofline": dict(hbm_roofline(scan_bytes, pre["scan_ms"], peaks, profile_traffic("scan_prefill262k")),
                              algorithmic="%.4g bytes per launch (10 B per token-channel)" % scan_bytes),
        "kernels_ms": {"scan": pre["scan_ms"], "attention": pre["attn_ms"]},
        "gpu_launches": pre["launches"],
        "clocks": pre["clocks"],
    }
    if "e2e_ms" in pre:
        line["e2e"] = {"value": tokens / (pre["e2e_ms"] * 1e-3), "unit": "tok/s",
                       "h2d_bytes_per_step": pre["h2d_bytes"], "d2h_bytes_per_step": pre["d2h_bytes"],
                       "call": "rat_mix_prefill with pinned-host inputs copied in and o copied out every step",
                       "pipelined": "copy-in of step i+1 and copy-out of step i-1 overlap step i (three streams, "
                                    "double-buffered device tensors); timed from the first copy-in to the last copy-out"}
    if dec:
        line["decode"] = {
            "metric": "decode tok/s (batch %d, H%d d%d D%d)" % (wd.decode_batch, wd.H, wd.d, wd.dil[0]),
            "workload": wd.name, "unit": "tok/s", "steps": dsteps,
            "by_ctx": [decode_entry(wd, r, dsteps, world, peaks,
                                    traffic=profile_traffic("decode_batch256", "decode_ctx%d" % r["ctx"]),
                                    cpu=cpu_entry(*oracle_decode_sample(wd, r["ctx"]),
                                                  "one batch entry's step (all heads) at position %d, repeated; "
                                                  "times the batch" % r["ctx"]) if cpu_ok else None)
                       for r in dec],
        }
    if cfgs:
        line["configs"] = {}
        for name, item in cfgs.items():
            wc, r = item[0], item[1]
            if name.startswith("prefill"):
                cpu = None
                if cpu_ok:
                    n_rows = 256
                    v, secs = oracle_sample(wc, n_rows)
                    cpu = cpu_entry(v, secs, "one head per head class: full scan + %d query rows spread over T; "
                                             "extrapolated to all heads" % n_rows)
                line["configs"][name] = prefill_entry(wc, r, args.steps, world, peaks, cpu)
            else:
                cpu = None
                if cpu_ok:
                    v, secs = oracle_decode_sample(wc, r["ctx"])
                    cpu = cpu_entry(v, secs, "one batch entry's step (all heads) at position %d, repeated; "
                                             "times the batch" % r["ctx"])
                e = decode_entry(wc, r, item[2], world, peaks, cpu=cpu)
                e["workload"] = wc.name + " decode batch %d" % wc.decode_batch
                line["configs"][name] = e
    if nxt:
        line["attention_variants"] = {}
        for name, r in att_var.items():
            t_from = w.T * 3 // 4 if name == "chunked" else 0
            Tv = RAGGED_T if name == "ragged" else w.T
            fl = sum(w.B * 4.0 * w.d * variant_pairs(Tv, w.dil[h], w.win[h], grid=name == "grid",
                                                     dedupe=name == "dedupe", t_from=t_from) for h in range(w.H))
            line["attention_variants"][name] = {
                "what": {"grid": "fixed-grid dilation (j mod D == D-1, plus t)",
                         "dedupe": "window part without the dilated set's keys",
                         "chunked": "last quarter of the prefill as a chunk (t0 = 3T/4) over the whole history",
                         "ragged": "T = %d, which D = 64 does not divide (two residue groups of %d and %d rows)"
                                   % (RAGGED_T, -(-RAGGED_T // 64), RAGGED_T // 64)}[name],
                "ms_per_launch": r["ms"], "value": w.B * (Tv - t_from) * world / (r["ms"] * 1e-3), "unit": "tok/s",
                "roofline": tensor_roofline(fl, r["ms"], peaks),
                "gpu_launches": r["launches"]}
        desc = {"grid_decode": "fixed-grid dilation, grid cache + window ring, ctx 4096",
                "paged_decode": "residue cache in 256-row pages (shuffled), ctx 4096",
                "topk_decode": "top-k blocks (Quest, block 64, K 16) over a dense cache, ctx 16384"}
        line["decode_variants"] = {
            name: {"what": desc[name], "value": wd.decode_batch * world / (r["ms"] * 1e-3), "unit": "tok/s",
                   "ms_per_step": r["ms"], "roofline": hbm_roofline(r["bytes"], r["ms"], peaks),
                   "gpu_launches": r["launches"]} for name, r in nxt.items()}
    if cpu_ok:
        v, secs = oracle_sample(w, args.cpu_rows)
        line["cpu_baseline"] = {"value": v, "unit": "tok/s", "cores": host_cores(), "kind": "oracle",
                                "sample": "head 0 of %d: full scan over T=%d + %d query rows spread over T "
                                          "(%.1f s); extrapolated to all heads" % (w.H, w.T, args.cpu_rows, secs)}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

"""The algorithmic work bench.py divides by (roofline numerators), on the CPU.

attn_pairs and decode_bytes count what the operator must touch; here they are
checked against brute-force enumeration of the key sets on small sizes, and
the profile-traffic reader against a synthetic summary.
"""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def brute_pairs(T, D, W):
    n = 0
    for t in range(T):
        n += sum(1 for j in range(t + 1) if (t - j) % D == 0)
        if W > 0:
            n += sum(1 for j in range(t + 1) if j >= t - W + 1)
    return n


@pytest.mark.parametrize("T,D,W", [(1, 1, 0), (7, 3, 0), (37, 4, 5), (64, 64, 64), (50, 7, 100), (100, 200, 3),
                                   (96, 1, 1)])
def test_attn_pairs_counts_every_unmasked_pair(T, D, W):
    assert bench.attn_pairs(T, D, W) == brute_pairs(T, D, W)


@pytest.mark.parametrize("t,D,W", [(0, 1, 0), (0, 4, 3), (1, 1, 0), (17, 4, 0), (17, 4, 5), (100, 7, 300),
                                   (4095, 16, 0), (4096, 64, 256)])
def test_decode_bytes_read_each_attended_row_once(t, D, W):
    # old cache rows a step at position t reads: its residue's rows before t,
    # then the window's rows before t (the new row comes from the state)
    B, H, d, elt = 3, 2, 128, 2
    rows = sum(1 for j in range(t) if (t - j) % D == 0) + (sum(1 for j in range(t) if j >= t - W + 1) if W else 0)
    per_token = H * d * (5 * elt + 16 + 2 * elt)   # q,k,v,g in, o out; fp32 state r+w; new row k,v
    assert bench.decode_bytes(B, H, d, t, [D] * H, [W] * H, elt) == B * (H * rows * 2 * d * elt + per_token)


def test_prefill_work_sums_heads():
    class W:
        B, T, H, d, dtype = 2, 40, 3, 64, "bf16"
        dil, win, recur = [1, 4, 9], [0, 5, 0], [0, 1, 1]
    flops, scan_bytes = bench.prefill_work(W)
    assert flops == sum(2 * 4 * 64 * brute_pairs(40, D, Wn) for D, Wn in zip(W.dil, W.win))
    assert scan_bytes == 2 * 2 * 40 * 64 * 10     # two recurrent heads, 10 bytes per (token, channel)


def test_profile_traffic_needs_the_captured_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel source\n")
    sha = hashlib.sha1(src.read_bytes()).hexdigest()[:12]
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k_case.md").write_text("traffic_bytes_per_launch[x]: 1.5e9 (source sha1 %s of k.cu)\n" % sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("k_case", "x") == 1.5e9
    assert bench.profile_traffic("k_case", "y") is None       # no such key
    assert bench.profile_traffic("missing") is None
    src.write_text("kernel source, changed\n")
    assert bench.profile_traffic("k_case", "x") is None       # the counters belong to older code


@pytest.mark.parametrize("t,block,K", [(0, 4, 2), (3, 4, 2), (4, 4, 2), (9, 4, 2), (40, 4, 2), (40, 4, 64),
                                       (16450, 64, 16)])
def test_topk_decode_bytes_read_the_kept_rows_and_the_candidates(t, block, K):
    B, H, d, elt = 2, 3, 128, 2
    c = t // block
    cand = list(range(1, c))
    kept = {0, c} | set(cand[:K])          # which K does not matter for the byte count
    rows = sum(1 for j in range(t) if j // block in kept)      # old rows; the new one is in registers
    per = len(cand) * 2 * d * 4 + rows * 2 * d * elt + d * (5 * elt + 16 + 2 * elt) + 2 * 2 * d * 4
    assert bench.topk_decode_bytes(B, H, d, t, block, K, elt) == B * H * per


@pytest.mark.parametrize("grid", [False, True])
@pytest.mark.parametrize("dedupe", [False, True])
@pytest.mark.parametrize("T,D,W", [(1, 1, 0), (37, 4, 5), (50, 7, 100), (64, 1, 8), (100, 9, 1), (90, 30, 61)])
def test_variant_pairs_count_the_reading_key_sets(grid, dedupe, T, D, W):
    n = 0
    for t in range(T):
        dil = {j for j in range(t + 1) if ((j % D == D - 1 or j == t) if grid else (t - j) % D == 0)}
        win = {j for j in range(t + 1) if W > 0 and j >= t - W + 1}
        n += len(dil) + len(win - dil if dedupe else win)
    assert bench.variant_pairs(T, D, W, grid=grid, dedupe=dedupe) == n
    # a chunk's rows alone: the whole minus the rows before it
    t_from = T // 3
    n_before = bench.variant_pairs(t_from, D, W, grid=grid, dedupe=dedupe) if t_from else 0.0
    assert bench.variant_pairs(T, D, W, grid=grid, dedupe=dedupe, t_from=t_from) == n - n_before
    if not grid and not dedupe:
        assert bench.attn_pairs(T, D, W) == n

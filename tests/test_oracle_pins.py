"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against a closed form, a special case that reduces
to a library routine (torch's scaled_dot_product_attention in float64), an
invariant, brute force over tiny inputs, or a hand-worked example stored under
tests/golden/.  Together they are chosen so that a dropped term, a swapped gate,
an off-by-one time index, a wrong dilation residue, a window off by one, or a
wrong merge fails at least one of them (tests/test_oracle_mutants.py plants such
mistakes in a copy of the oracle and checks that they are caught).

Sources: "RAT+: Train Dense, Infer Sparse" Abstract, Figure 1(a)/(c), Figure 2;
"Augmenting Attention with Exponentially Decaying Memory" section 2.1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
rng = np.random.default_rng(12345)


def sig(z):
    return 1.0 / (1.0 + np.exp(-z))


# ----------------------------------------------------------------------------- scan


def test_scan_golden_worked_example():
    j = json.load(open(os.path.join(GOLDEN, "scan_worked_example.json")))
    x = np.array(j["x"]).reshape(1, -1, 1, 1)
    g = np.array(j["g"]).reshape(1, -1, 1, 1)
    init = np.array([[[j["init"]]]])
    out, final = oracle.scan(x, g, init)
    np.testing.assert_allclose(out.ravel(), j["expected"], rtol=0, atol=j["tol"])
    assert abs(final.ravel()[0] - j["expected"][-1]) < j["tol"]


@pytest.mark.parametrize("gval", [-1.3, 0.0, 2.0, 4.5])
def test_scan_constant_gate_geometric_sum(gval):
    # constant a: s_t = (1-a) sum_{u<=t} a^(t-u) x_u + a^(t+1) s_{-1}
    B, T, H, d = 2, 37, 3, 5
    x = rng.standard_normal((B, T, H, d))
    init = rng.standard_normal((B, H, d))
    g = np.full_like(x, gval)
    out, final = oracle.scan(x, g, init)
    a = sig(gval)
    expect = np.empty_like(x)
    for t in range(T):
        w = (1 - a) * a ** (t - np.arange(t + 1))           # weight of x_u, u = 0..t
        expect[:, t] = np.einsum("u,buhc->bhc", w, x[:, : t + 1]) + a ** (t + 1) * init
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(final, expect[:, -1], rtol=1e-12, atol=1e-12)


def test_scan_constant_input_closed_form():
    # constant x = X, constant a: s_t = X (1 - a^(t+1)) + a^(t+1) s_{-1}
    T = 50
    X, I, gval = 1.75, -0.5, 1.2
    x = np.full((1, T, 1, 1), X)
    out, _ = oracle.scan(x, np.full_like(x, gval), np.array([[[I]]]))
    a = sig(gval)
    t = np.arange(T)
    np.testing.assert_allclose(out.ravel(), X * (1 - a ** (t + 1)) + a ** (t + 1) * I, rtol=1e-13, atol=1e-13)


def test_scan_time_varying_gate_explicit_solution():
    # unrolled solution of the recurrence:
    #   s_t = sum_{u<=t} (1-a_u) prod_{w=u+1..t} a_w x_u + prod_{w=0..t} a_w s_{-1}
    B, T, H, d = 1, 12, 2, 3
    x = rng.standard_normal((B, T, H, d))
    g = 2.0 * rng.standard_normal((B, T, H, d))
    init = rng.standard_normal((B, H, d))
    out, _ = oracle.scan(x, g, init)
    a = sig(g)
    expect = np.zeros_like(x)
    for t in range(T):
        acc = np.prod(a[:, 0 : t + 1], axis=1) * init
        for u in range(t + 1):
            acc = acc + (1 - a[:, u]) * np.prod(a[:, u + 1 : t + 1], axis=1) * x[:, u]
        expect[:, t] = acc
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-13)


def test_scan_gate_limits():
    B, T, H, d = 1, 9, 2, 4
    x = rng.standard_normal((B, T, H, d))
    init = rng.standard_normal((B, H, d))
    # a -> 0: no memory, s_t = x_t
    out, _ = oracle.scan(x, np.full_like(x, -60.0), init)
    np.testing.assert_allclose(out, x, rtol=0, atol=1e-20)
    # a == 1 in double: the state never moves from s_{-1}
    out, final = oracle.scan(x, np.full_like(x, 60.0), init)
    assert np.array_equal(out, np.broadcast_to(init[:, None], out.shape))
    assert np.array_equal(final, init)


def test_scan_chunked_equals_one_shot():
    # carrying the final state into the next chunk reproduces the one-shot scan
    B, T, H, d = 2, 40, 2, 3
    x = rng.standard_normal((B, T, H, d))
    g = 1.0 + rng.standard_normal((B, T, H, d))
    full, ffull = oracle.scan(x, g)
    o1, f1 = oracle.scan(x[:, :17], g[:, :17])
    o2, f2 = oracle.scan(x[:, 17:], g[:, 17:], f1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), full, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(f2, ffull, rtol=1e-14, atol=1e-14)


def test_scan_recur_off_is_identity():
    B, T, H, d = 1, 10, 3, 2
    x = rng.standard_normal((B, T, H, d))
    g = rng.standard_normal((B, T, H, d))
    out, final = oracle.scan(x, g, recur=[1, 0, 1])
    assert np.array_equal(out[:, :, 1], x[:, :, 1])
    assert np.array_equal(final[:, 1], x[:, -1, 1])
    assert not np.allclose(out[:, :, 0], x[:, :, 0])


def test_scan_zero_length():
    x = np.zeros((1, 0, 1, 2))
    init = np.array([[[0.5, -1.0]]])
    out, final = oracle.scan(x, x, init)
    assert out.shape == (1, 0, 1, 2)
    assert np.array_equal(final, init)


# ------------------------------------------------------------------------ attention


def sdpa_causal(q, k, v, scale, mask=None):
    """torch SDPA in float64 on [T, d] operands of one head."""
    q, k, v = (torch.from_numpy(np.ascontiguousarray(a))[None, None] for a in (q, k, v))
    if mask is None:
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
    else:
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(mask)[None, None], scale=scale)
    return o[0, 0].numpy()


def rand_qkv(B, T, H, d):
    return (rng.standard_normal((B, T, H, d)) for _ in range(3))


def test_attention_golden_worked_example():
    j = json.load(open(os.path.join(GOLDEN, "attn_worked_example.json")))
    shp = (1, 3, 1, 1)
    q, k, v = (np.array(j[n]).reshape(shp) for n in ("q", "k", "v"))
    dil, win = [j["D"]], [j["W"]]
    e, tol = j["expected"], j["tol"]
    o, lse = oracle.attn_rows(q, k, v, dil, win, [[0, 0, 2]], parts=1, scale=j["scale"])
    assert abs(o[0, 0] - e["t2"]["o_dil"]) < tol and abs(lse[0] - e["t2"]["lse_dil"]) < tol
    o, lse = oracle.attn_rows(q, k, v, dil, win, [[0, 0, 2]], parts=2, scale=j["scale"])
    assert abs(o[0, 0] - e["t2"]["o_win"]) < tol and abs(lse[0] - e["t2"]["lse_win"]) < tol
    o, lse = oracle.attn_rows(q, k, v, dil, win, [[0, 0, 0], [0, 0, 1], [0, 0, 2]], parts=3, scale=j["scale"])
    for i, key in enumerate(("t0", "t1", "t2")):
        assert abs(o[i, 0] - e[key]["o"]) < tol, key
        assert abs(lse[i] - e[key]["lse"]) < tol, key


@pytest.mark.parametrize("T,d", [(1, 8), (33, 16), (70, 7)])
def test_dense_causal_equals_sdpa(T, d):
    # D = 1, no window, a = 0 (keys/values unaugmented): plain causal attention
    B, H = 2, 2
    q, k, v = rand_qkv(B, T, H, d)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attention(q, k, v, [1] * H, [0] * H)
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(o[b, :, h], sdpa_causal(q[b, :, h], k[b, :, h], v[b, :, h], scale),
                                       rtol=1e-12, atol=1e-12)
            s = scale * q[b, :, h] @ k[b, :, h].T
            s[np.triu_indices(T, 1)] = -np.inf
            ref = torch.logsumexp(torch.from_numpy(s), dim=-1).numpy()
            np.testing.assert_allclose(lse[b, h], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T,D", [(64, 4), (50, 7), (5, 8), (31, 2), (40, 40)])
def test_dilated_equals_interleaved_subsequences(T, D):
    # dilation D == D independent dense causal attentions over r, r+D, r+2D, ...
    B, H, d = 1, 2, 6
    q, k, v = rand_qkv(B, T, H, d)
    scale = 0.37
    o, _ = oracle.attention(q, k, v, [D] * H, [0] * H, scale=scale)
    expect = np.empty_like(o)
    for h in range(H):
        for r in range(min(D, T)):
            idx = np.arange(r, T, D)
            expect[0, idx, h] = sdpa_causal(q[0, idx, h], k[0, idx, h], v[0, idx, h], scale)
    np.testing.assert_allclose(o, expect, rtol=1e-12, atol=1e-12)


def test_window_covering_everything_is_dense_causal():
    B, T, H, d = 1, 45, 1, 8
    q, k, v = rand_qkv(B, T, H, d)
    for W in (T, T + 5):
        o, _ = oracle.attention(q, k, v, [3], [W], parts=2)
        np.testing.assert_allclose(o[0, :, 0], sdpa_causal(q[0, :, 0], k[0, :, 0], v[0, :, 0], 1 / math.sqrt(d)),
                                   rtol=1e-12, atol=1e-12)


def test_window_of_one_is_own_value():
    B, T, H, d = 1, 20, 2, 4
    q, k, v = rand_qkv(B, T, H, d)
    o, lse = oracle.attention(q, k, v, [5, 5], [1, 1], parts=2, scale=0.5)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, 0.5 * np.einsum("bthc,bthc->bht", q, k), rtol=1e-13, atol=1e-13)


def test_window_extent_by_band():
    # window W: exactly the W keys t-W+1..t (band mask handed to SDPA)
    B, T, H, d, W = 1, 30, 1, 5, 6
    q, k, v = rand_qkv(B, T, H, d)
    o, _ = oracle.attention(q, k, v, [4], [W], parts=2)
    i, j = np.meshgrid(np.arange(T), np.arange(T), indexing="ij")
    band = (j <= i) & (j > i - W)
    np.testing.assert_allclose(o[0, :, 0], sdpa_causal(q[0, :, 0], k[0, :, 0], v[0, :, 0], 1 / math.sqrt(d), band),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T,D,W", [(40, 4, 6), (33, 5, 1), (20, 3, 40), (17, 1, 4)])
def test_merge_is_one_softmax_over_both_sets(T, D, W):
    # brute force: one softmax over the concatenated multiset of both key sets
    B, H, d = 1, 1, 5
    q, k, v = rand_qkv(B, T, H, d)
    scale = 0.6
    o, lse = oracle.attention(q, k, v, [D], [W], parts=3, scale=scale)
    for t in range(T):
        keys = [j for j in range(t + 1) if (t - j) % D == 0] + [j for j in range(max(0, t - W + 1), t + 1)]
        z = torch.from_numpy(scale * k[0, keys, 0] @ q[0, t, 0])
        p = torch.softmax(z, dim=0).numpy()
        np.testing.assert_allclose(o[0, t, 0], p @ v[0, keys, 0], rtol=1e-12, atol=1e-12)
        assert abs(lse[0, 0, t] - torch.logsumexp(z, 0).item()) < 1e-12


def test_huge_scores_select_the_best_key():
    # scale -> infinity: each row's softmax collapses onto its largest-score key
    # (no overflow: the max is taken out before exponentiating)
    B, T, H, d = 1, 40, 1, 8
    q, k, v = rand_qkv(B, T, H, d)
    o, lse = oracle.attention(q, k, v, [3], [5], scale=1e6)
    for t in range(T):
        keys = sorted({j for j in range(t + 1) if (t - j) % 3 == 0} | set(range(max(0, t - 4), t + 1)))
        z = k[0, keys, 0] @ q[0, t, 0]
        best = keys[int(np.argmax(z))]
        np.testing.assert_allclose(o[0, t, 0], v[0, best, 0], rtol=0, atol=1e-9)
        assert np.isfinite(lse[0, 0, t])


def test_first_row_and_convex_hull():
    B, T, H, d = 2, 30, 2, 6
    q, k, v = rand_qkv(B, T, H, d)
    o, lse = oracle.attention(q, k, v, [3, 7], [4, 0])
    np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=0, atol=1e-14)
    for t in range(T):
        lo = v[:, : t + 1].min(axis=1)
        hi = v[:, : t + 1].max(axis=1)
        assert np.all(o[:, t] >= lo - 1e-12) and np.all(o[:, t] <= hi + 1e-12)


# -------------------------------------------------- fixed-grid dilation (comparison)
# The fixed-grid reading: query t's dilated part takes the keys j <= t with
# j mod D == D - 1 (one per chunk of D tokens, shared by all queries) plus t.


@pytest.mark.parametrize("T", [1, 19])
def test_grid_with_d_1_is_dense_causal(T):
    B, H, d = 1, 2, 6
    q, k, v = rand_qkv(B, T, H, d)
    o, _ = oracle.attention(q, k, v, [1] * H, [0] * H, grid=True)
    for h in range(H):
        np.testing.assert_allclose(o[0, :, h], sdpa_causal(q[0, :, h], k[0, :, h], v[0, :, h], 1 / math.sqrt(d)),
                                   rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T,D", [(37, 3), (37, 5), (20, 8), (9, 12)])
def test_grid_equals_masked_sdpa(T, D):
    # brute force: SDPA with the boolean mask of the grid set
    B, H, d = 1, 1, 7
    q, k, v = rand_qkv(B, T, H, d)
    scale = 0.45
    o, _ = oracle.attention(q, k, v, [D], [0], parts=1, scale=scale, grid=True)
    i, j = np.meshgrid(np.arange(T), np.arange(T), indexing="ij")
    mask = (j <= i) & ((j % D == D - 1) | (j == i))
    np.testing.assert_allclose(o[0, :, 0], sdpa_causal(q[0, :, 0], k[0, :, 0], v[0, :, 0], scale, mask),
                               rtol=1e-12, atol=1e-12)


def test_grid_rows_on_the_grid_equal_the_residue_reading():
    # for t with t mod D == D - 1 both readings select the same keys
    B, T, H, d = 1, 50, 2, 5
    q, k, v = rand_qkv(B, T, H, d)
    dil = [4, 7]
    rows = [(0, h, t) for h in range(H) for t in range(T) if t % dil[h] == dil[h] - 1]
    og, lg = oracle.attn_rows(q, k, v, dil, [0, 0], rows, parts=1, grid=True)
    orr, lr = oracle.attn_rows(q, k, v, dil, [0, 0], rows, parts=1)
    np.testing.assert_allclose(og, orr, rtol=0, atol=0)
    np.testing.assert_allclose(lg, lr, rtol=0, atol=0)


def test_grid_rows_before_the_first_grid_key_see_only_themselves():
    B, T, H, d, D = 1, 6, 1, 4, 8
    q, k, v = rand_qkv(B, T, H, d)
    o, lse = oracle.attention(q, k, v, [D], [0], parts=1, scale=0.5, grid=True)
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], 0.5 * np.einsum("tc,tc->t", q[0, :, 0], k[0, :, 0]), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("T,D,W", [(40, 4, 6), (23, 6, 2)])
def test_grid_merge_is_one_softmax_over_both_sets(T, D, W):
    B, H, d = 1, 1, 5
    q, k, v = rand_qkv(B, T, H, d)
    scale = 0.6
    o, lse = oracle.attention(q, k, v, [D], [W], parts=3, scale=scale, grid=True)
    for t in range(T):
        keys = [j for j in range(t + 1) if j % D == D - 1 or j == t] + [j for j in range(max(0, t - W + 1), t + 1)]
        z = torch.from_numpy(scale * k[0, keys, 0] @ q[0, t, 0])
        p = torch.softmax(z, dim=0).numpy()
        np.testing.assert_allclose(o[0, t, 0], p @ v[0, keys, 0], rtol=1e-12, atol=1e-12)
        assert abs(lse[0, 0, t] - torch.logsumexp(z, 0).item()) < 1e-12


# ------------------------------------------------- dedupe variant of the merge
# With dedupe, a key in both parts counts once: the merge is one softmax over
# the union of the dilated and window sets (the default counts the multiset).


@pytest.mark.parametrize("T,D,W,grid", [(40, 4, 6, False), (33, 5, 1, False), (20, 3, 40, False),
                                        (29, 4, 9, True), (25, 6, 3, True)])
def test_dedupe_merge_is_one_softmax_over_the_union(T, D, W, grid):
    B, H, d = 1, 1, 5
    q, k, v = rand_qkv(B, T, H, d)
    scale = 0.6
    o, lse = oracle.attention(q, k, v, [D], [W], parts=3, scale=scale, grid=grid, dedupe=True)
    for t in range(T):
        dil_set = {j for j in range(t + 1) if ((j % D == D - 1 or j == t) if grid else (t - j) % D == 0)}
        keys = sorted(dil_set | set(range(max(0, t - W + 1), t + 1)))
        z = torch.from_numpy(scale * k[0, keys, 0] @ q[0, t, 0])
        p = torch.softmax(z, dim=0).numpy()
        np.testing.assert_allclose(o[0, t, 0], p @ v[0, keys, 0], rtol=1e-12, atol=1e-12)
        assert abs(lse[0, 0, t] - torch.logsumexp(z, 0).item()) < 1e-12


def test_dedupe_with_d_1_is_dense_causal():
    # every window key is already a dilated key at D = 1
    B, T, H, d = 1, 26, 1, 6
    q, k, v = rand_qkv(B, T, H, d)
    o, _ = oracle.attention(q, k, v, [1], [5], dedupe=True)
    np.testing.assert_allclose(o[0, :, 0], sdpa_causal(q[0, :, 0], k[0, :, 0], v[0, :, 0], 1 / math.sqrt(d)),
                               rtol=1e-12, atol=1e-12)


def test_dedupe_without_window_changes_nothing():
    B, T, H, d = 1, 30, 2, 4
    q, k, v = rand_qkv(B, T, H, d)
    a = oracle.attention(q, k, v, [3, 7], [0, 0])
    b = oracle.attention(q, k, v, [3, 7], [0, 0], dedupe=True)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# --------------------------------------------------------------------------- top-k blocks


def topk_rows(T, H=1, B=1):
    return [(b, h, t) for b in range(B) for h in range(H) for t in range(T)]


def masked_rows(q, k, v, keysets, scale):
    """Softmax attention of row t of q over the explicit key set keysets[t]."""
    out, lses = [], []
    for t, keys in enumerate(keysets):
        keys = sorted(keys)
        z = torch.from_numpy(scale * k[keys] @ q[t])
        out.append(torch.softmax(z, dim=0).numpy() @ v[keys])
        lses.append(torch.logsumexp(z, 0).item())
    return np.array(out), np.array(lses)


@pytest.mark.parametrize("mode", ["quest", "moba"])
@pytest.mark.parametrize("T,bs", [(29, 4), (16, 16), (7, 3)])
def test_topk_with_every_block_kept_is_dense_causal(mode, T, bs):
    B, H, d = 1, 2, 5
    q, k, v = rand_qkv(B, T, H, d)
    rows = topk_rows(T, H)
    o, lse = oracle.attn_rows_topk(q, k, v, bs, T, mode, rows)
    for h in range(H):
        ref = sdpa_causal(q[0, :, h], k[0, :, h], v[0, :, h], 1 / math.sqrt(d))
        np.testing.assert_allclose(o[h * T:(h + 1) * T], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", ["quest", "moba"])
def test_topk_with_k_0_keeps_first_and_local_block(mode):
    B, T, H, d, bs = 1, 23, 1, 4, 5
    q, k, v = rand_qkv(B, T, H, d)
    o, lse = oracle.attn_rows_topk(q, k, v, bs, 0, mode, topk_rows(T), scale=0.7)
    sets = [[j for j in range(t + 1) if j < bs or j >= (t // bs) * bs] for t in range(T)]
    ro, rl = masked_rows(q[0, :, 0], k[0, :, 0], v[0, :, 0], sets, 0.7)
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", ["quest", "moba"])
@pytest.mark.parametrize("K", [1, 3])
def test_topk_with_blocks_of_one_key_is_top_k_keys(mode, K):
    # a one-key block has kmin = kmax = mean = k, so both scores are q.k and the
    # selection is the K largest dot products among keys 1 .. t-1
    B, T, H, d = 1, 19, 1, 6
    q, k, v = rand_qkv(B, T, H, d)
    o, lse = oracle.attn_rows_topk(q, k, v, 1, K, mode, topk_rows(T))
    qq, kk = q[0, :, 0], k[0, :, 0]
    sets = []
    for t in range(T):
        cand = list(range(1, t))
        best = sorted(cand, key=lambda j: -float(kk[j] @ qq[t]))[:K]
        sets.append(set([0, t] + best))
    ro, rl = masked_rows(qq, kk, v[0, :, 0], sets, 1 / math.sqrt(d))
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_topk_quest_and_moba_worked_example():
    # blocks of 2 over T = 8 (blocks 0..3); rows 6 and 7 sit in block 3, one
    # candidate (K = 1) among blocks 1 and 2, d = 2:
    #   block 1 keys (-3, 0), (5, 0): mean (1, 0);   block 2 keys (-2, 1) twice
    #   row 7, q = (-1, 0.5): Quest bound  block1 = 3 + 0 = 3,  block2 = 2 + 0.5 = 2.5 -> block 1
    #                        MoBA mean     block1 = -1,        block2 = 2.5        -> block 2
    #   row 6, q = (1, 0):    Quest bound  block1 = 5,          block2 = -2         -> block 1
    #                        MoBA mean     block1 = 1,          block2 = -2         -> block 1
    k = np.zeros((1, 8, 1, 2))
    k[0, :, 0] = [[0.3, -0.2], [0.1, 0.4], [-3, 0], [5, 0], [-2, 1], [-2, 1], [0.2, 0.2], [-0.1, 0.3]]
    q = np.zeros((1, 8, 1, 2))
    q[0, 6, 0] = [1, 0]
    q[0, 7, 0] = [-1, 0.5]
    v = rng.standard_normal((1, 8, 1, 2))
    rows = [(0, 0, 6), (0, 0, 7)]
    expect = {"quest": [{0, 1, 2, 3, 6}, {0, 1, 2, 3, 6, 7}],
              "moba": [{0, 1, 2, 3, 6}, {0, 1, 4, 5, 6, 7}]}
    for mode, sets in expect.items():
        o, lse = oracle.attn_rows_topk(q, k, v, 2, 1, mode, rows, scale=0.5)
        ro, rl = masked_rows(q[0, 6:, 0], k[0, :, 0], v[0, :, 0], sets, 0.5)
        np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", ["quest", "moba"])
def test_topk_equal_scores_go_to_the_lower_block(mode):
    B, T, H, d, bs = 1, 12, 1, 3, 3
    q, k, v = rand_qkv(B, T, H, d)
    k[0, 6:9] = k[0, 3:6]          # blocks 1 and 2 hold the same keys
    o, _ = oracle.attn_rows_topk(q, k, v, bs, 1, mode, [(0, 0, 11)])
    ro, _ = masked_rows(q[0, 11:, 0], k[0, :, 0], v[0, :, 0], [{0, 1, 2, 3, 4, 5, 9, 10, 11}], 1 / math.sqrt(d))
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", ["quest", "moba"])
def test_topk_selection_is_what_the_rows_attend(mode):
    # the exported selection and the attention rows agree: each row equals a
    # softmax over the first block, its own block and the selected ones
    B, T, H, d, bs, K = 1, 41, 1, 4, 4, 2
    q, k, v = rand_qkv(B, T, H, d)
    rows = topk_rows(T)
    o, lse = oracle.attn_rows_topk(q, k, v, bs, K, mode, rows)
    sel, gap = oracle.topk_select(q, k, bs, K, mode, rows)
    sets = []
    for t in range(T):
        blocks = {0, t // bs} | {int(x) for x in sel[t] if x >= 0}
        sets.append({j for j in range(t + 1) if j // bs in blocks})
        ncand = max(0, t // bs - 1)
        assert (sel[t] >= 0).sum() == min(K, ncand)
        assert all(1 <= x < t // bs for x in sel[t] if x >= 0)
    ro, rl = masked_rows(q[0, :, 0], k[0, :, 0], v[0, :, 0], sets, 1 / math.sqrt(d))
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_topk_selection_with_blocks_of_one_key_sorts_dot_products():
    # one-key blocks: picks in descending q.k among keys 1 .. t-1, and the gap
    # is the K-th largest minus the (K+1)-th
    B, T, H, d, K = 1, 23, 1, 5, 3
    q, k, _ = rand_qkv(B, T, H, d)
    sel, gap = oracle.topk_select(q, k, 1, K, "moba", topk_rows(T))
    for t in range(T):
        dots = {j: float(k[0, j, 0] @ q[0, t, 0]) for j in range(1, t)}
        order = sorted(dots, key=lambda j: -dots[j])
        want = order[:K] + [-1] * (K - len(order[:K]))
        assert list(sel[t]) == want
        if len(order) > K:
            assert abs(gap[t] - (dots[order[K - 1]] - dots[order[K]])) < 1e-12
        else:
            assert gap[t] == np.inf


def test_topk_selection_worked_example():
    # the hand-worked blocks of test_topk_quest_and_moba_worked_example:
    #   row 7: Quest 3 vs 2.5 -> picks block 1, gap 0.5; MoBA 2.5 vs -1 -> block 2, gap 3.5
    #   row 6: Quest 5 vs -2 -> block 1, gap 7;         MoBA 1 vs -2 -> block 1, gap 3
    k = np.zeros((1, 8, 1, 2))
    k[0, :, 0] = [[0.3, -0.2], [0.1, 0.4], [-3, 0], [5, 0], [-2, 1], [-2, 1], [0.2, 0.2], [-0.1, 0.3]]
    q = np.zeros((1, 8, 1, 2))
    q[0, 6, 0] = [1, 0]
    q[0, 7, 0] = [-1, 0.5]
    rows = [(0, 0, 6), (0, 0, 7)]
    sel, gap = oracle.topk_select(q, k, 2, 1, "quest", rows)
    assert sel.tolist() == [[1], [1]] and np.allclose(gap, [7.0, 0.5], rtol=0, atol=1e-12)
    sel, gap = oracle.topk_select(q, k, 2, 1, "moba", rows)
    assert sel.tolist() == [[1], [2]] and np.allclose(gap, [3.0, 3.5], rtol=0, atol=1e-12)


def test_topk_invalid_arguments_are_rejected():
    q, k, v = rand_qkv(1, 4, 1, 2)
    for bs, K, rows in [(0, 1, [(0, 0, 1)]), (2, -1, [(0, 0, 1)]), (2, 1, [(0, 0, 4)])]:
        with pytest.raises(ValueError):
            oracle.attn_rows_topk(q, k, v, bs, K, "quest", rows)


# --------------------------------------------------------------------------- decode


@pytest.mark.parametrize("heads", [dict(dil=[4, 1, 3], win=[0, 0, 5], recur=[1, 0, 1])])
def test_decode_equals_last_prefill_row(heads):
    # decode at position t after a prefill of t tokens == row t of a prefill of t+1
    B, T, H, d = 2, 23, 3, 4
    q, k, v = rand_qkv(B, T + 1, H, d)
    g = 1.0 + rng.standard_normal((B, T + 1, H, d))
    dil, win, recur = heads["dil"], heads["win"], heads["recur"]
    full = oracle.mix_prefill(q, k, v, g, dil, win, recur)
    pre = oracle.mix_prefill(q[:, :T], k[:, :T], v[:, :T], g[:, :T], dil, win, recur)
    cap = T + 4
    hist_k = np.zeros((B, cap, H, d))
    hist_v = np.zeros((B, cap, H, d))
    hist_k[:, :T], hist_v[:, :T] = pre["kt"], pre["vt"]
    sk, sv = pre["final_k"].copy(), pre["final_v"].copy()
    o, lse = oracle.decode_step(q[:, T], k[:, T], v[:, T], g[:, T], sk, sv, hist_k, hist_v,
                                [T] * B, dil, win, recur)
    np.testing.assert_allclose(o, full["o"][:, T], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, full["lse"][:, :, T], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sk, full["final_k"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(sv, full["final_v"], rtol=1e-13, atol=1e-13)


def test_decode_steps_replay_prefill():
    # several decode steps from an empty history reproduce every prefill row
    B, T, H, d = 1, 9, 2, 3
    q, k, v = rand_qkv(B, T, H, d)
    g = rng.standard_normal((B, T, H, d))
    dil, win, recur = [2, 3], [3, 0], [1, 1]
    full = oracle.mix_prefill(q, k, v, g, dil, win, recur)
    hk, hv = np.zeros((B, T, H, d)), np.zeros((B, T, H, d))
    sk, sv = np.zeros((B, H, d)), np.zeros((B, H, d))
    for t in range(T):
        o, _ = oracle.decode_step(q[:, t], k[:, t], v[:, t], g[:, t], sk, sv, hk, hv, [t] * B, dil, win, recur)
        np.testing.assert_allclose(o, full["o"][:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hk, full["kt"], rtol=1e-13, atol=1e-13)


def test_invalid_arguments_are_rejected():
    q = np.zeros((1, 4, 1, 2))
    with pytest.raises(ValueError):
        oracle.attn_rows(q, q, q, [0], [0], [[0, 0, 1]])          # D < 1
    with pytest.raises(ValueError):
        oracle.attn_rows(q, q, q, [1], [0], [[0, 0, 4]])          # t out of range
    with pytest.raises(ValueError):
        oracle.attn_rows(q, q, q, [1], [0], [[0, 0, 1]], parts=2)  # no window to take

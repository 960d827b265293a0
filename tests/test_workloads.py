"""The seeded input generators against the input recipe (CPU only).

q, k, v ~ N(0, 1) and gate logits ~ N(mu, 1), drawn in that order from one
seeded generator, cast to the workload's dtype; the named workloads carry the
sizes the benchmark and the parity tests use.
"""
import torch

import workloads as wl


def test_prefill_inputs_follow_the_recipe():
    q, k, v, g = wl.prefill_inputs(2, 4096, 4, 64, 2.0, torch.float32, seed=3)
    for x in (q, k, v, g):
        assert x.shape == (2, 4096, 4, 64) and x.dtype == torch.float32
    for x in (q, k, v):
        assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    assert abs(g.mean().item() - 2.0) < 0.01 and abs(g.std().item() - 1.0) < 0.01


def test_inputs_are_seeded_and_cast():
    a = wl.prefill_inputs(1, 64, 2, 64, 1.0, torch.bfloat16, seed=7)
    b = wl.prefill_inputs(1, 64, 2, 64, 1.0, torch.bfloat16, seed=7)
    c = wl.prefill_inputs(1, 64, 2, 64, 1.0, torch.bfloat16, seed=8)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not torch.equal(a[0], c[0])
    assert all(x.dtype == torch.bfloat16 for x in a)
    # the bf16 tensors are the fp32 draws rounded
    f = wl.prefill_inputs(1, 64, 2, 64, 1.0, torch.float32, seed=7)
    assert all(torch.equal(x.float(), y.to(torch.bfloat16).float()) for x, y in zip(a, f))


def test_token_inputs_are_one_position():
    q, k, v, g = wl.token_inputs(3, 4, 128, 2.0, torch.bfloat16, seed=1)
    full = wl.prefill_inputs(3, 1, 4, 128, 2.0, torch.bfloat16, seed=1)
    for x, y in zip((q, k, v, g), full):
        assert x.shape == (3, 4, 128) and torch.equal(x, y.reshape(3, 4, 128))


def test_named_workloads():
    w = wl.PREFILL_262K
    assert (w.B, w.T, w.H, w.d, w.dtype) == (1, 262144, 16, 128, "bf16")
    assert set(w.dil) == {64} and set(w.win) == {512} and all(w.recur)
    d = wl.DECODE_D16
    assert (d.decode_batch, d.H, d.d) == (256, 16, 128) and set(d.dil) == {16}
    assert d.decode_ctx == [4096, 16384, 32768]
    t = wl.TINY_F32
    assert (t.B, t.T, t.H, t.d, t.dtype) == (1, 256, 2, 64, "f32") and set(t.dil) == {4}

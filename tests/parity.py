"""Shared helpers of the GPU parity tests: tolerances, comparisons, row sampling.

Tolerances (the operator's stated bar): fp32 operands -> max-abs error <= 1e-4;
bf16 operands -> relative L2 error <= 1e-2, both against the fp64 CPU oracle.
"""
import numpy as np
import torch

TOL_F32_MAXABS = 1e-4
TOL_BF16_RELL2 = 1e-2


def f64(t):
    """torch tensor (any device / dtype) -> numpy float64."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    return float(np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def max_abs(got, ref):
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64)))) if np.size(ref) else 0.0


def assert_close(got, ref, dtype, what=""):
    """The operator's bar: max-abs 1e-4 for fp32, relative L2 1e-2 for bf16."""
    got = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    assert got.shape == np.shape(ref), (what, got.shape, np.shape(ref))
    assert np.all(np.isfinite(got)), what + ": non-finite values"
    if dtype == torch.float32:
        e = max_abs(got, ref)
        assert e <= TOL_F32_MAXABS, "%s: max-abs %.3g > %.1g" % (what, e, TOL_F32_MAXABS)
    else:
        e = rel_l2(got, ref)
        assert e <= TOL_BF16_RELL2, "%s: rel-L2 %.3g > %.1g" % (what, e, TOL_BF16_RELL2)
    return e


def sample_rows(T, D, W, n_random=48, seed=0):
    """Query positions that cover the edges: t=0, t<D, residue and window
    boundaries, the last rows, plus a seeded random spread."""
    cand = {0, 1, 2, D - 1, D, D + 1, 2 * D - 1, 2 * D, W - 1, W, W + 1, T // 2, T - D - 1, T - D, T - 2, T - 1,
            128, 127, 129, 255, 256}
    rng = np.random.default_rng(seed)
    cand |= set(rng.integers(0, T, size=n_random).tolist())
    return sorted(t for t in cand if 0 <= t < T)

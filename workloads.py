"""Seeded synthetic workloads for the RAT+ temporal-mixing operator.

This module only draws random inputs and names the workload shapes.  It holds
none of the operator's arithmetic, so both the CPU oracle's tests and the CUDA
path's tests and benchmark can use it without sharing any computation.

Shapes follow the efficiency study of "RAT+: Train Dense, Infer Sparse --
Recurrence Augmented Attention for Dilated Inference" (Figure 2: prefill of 262K
tokens, decode at batch 256 / 128 for the two hidden sizes, 16 heads of 128 for
hidden 2048 and 32 heads of 128 for hidden 4096).  Values: q, k, v ~ N(0, 1) and
gate logits ~ N(mu, 1) per channel and position, drawn in the order q, k, v, g
from one torch generator seeded with `seed`, in fp32, then cast to the storage
dtype.  Layout [B, T, H, d], d fastest.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass
class Workload:
    name: str
    B: int
    T: int
    H: int
    d: int
    dtype: str                    # "f32" or "bf16"
    dil: List[int]
    win: List[int]
    recur: List[int]
    gate_mean: float
    decode_batch: int = 0
    decode_ctx: List[int] = field(default_factory=list)
    decode_steps: int = 0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


def _uniform(H, D, W, R):
    return dict(dil=[D] * H, win=[W] * H, recur=[R] * H)


# The five workloads of the operator study.
TINY_F32 = Workload("tiny-f32 B1 H2 d64 T256 D4", 1, 256, 2, 64, "f32", gate_mean=2.0,
                    **_uniform(2, 4, 0, 1))
PREFILL_16K = Workload("prefill-bf16 B1 H16 d128 T16384 D16", 1, 16384, 16, 128, "bf16",
                       gate_mean=2.0, **_uniform(16, 16, 0, 1))
PREFILL_262K = Workload("prefill-bf16 B1 H16 d128 T262144 D64 W512", 1, 262144, 16, 128, "bf16",
                        gate_mean=2.0, **_uniform(16, 64, 512, 1))
DECODE_D16 = Workload("decode-bf16 batch256 H16 d128 D16", 256, 0, 16, 128, "bf16", gate_mean=2.0,
                      decode_batch=256, decode_ctx=[4096, 16384, 32768], decode_steps=1024,
                      **_uniform(16, 16, 0, 1))
HYBRID = Workload("hybrid-bf16 B4 H32 d128 T65536 (4 dense + 28 D64 W256)", 4, 65536, 32, 128, "bf16",
                  gate_mean=3.0, dil=[1] * 4 + [64] * 28, win=[0] * 4 + [256] * 28,
                  recur=[0] * 4 + [1] * 28, decode_batch=128, decode_ctx=[65536], decode_steps=256)

ALL = [TINY_F32, PREFILL_16K, PREFILL_262K, DECODE_D16, HYBRID]


def make_generator(device, seed: int) -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return gen


def prefill_inputs(B, T, H, d, gate_mean, dtype=torch.bfloat16, device="cpu", seed=0):
    """(q, k, v, g), each [B, T, H, d] in `dtype`, drawn in that order."""
    gen = make_generator(device, seed)
    shape = (B, T, H, d)
    out = []
    for mean in (0.0, 0.0, 0.0, gate_mean):
        x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        if mean:
            x.add_(mean)
        out.append(x.to(dtype))
    return tuple(out)


def token_inputs(B, H, d, gate_mean, dtype=torch.bfloat16, device="cpu", seed=0):
    """(q, k, v, g) of one new token per batch entry, each [B, H, d]."""
    q, k, v, g = prefill_inputs(B, 1, H, d, gate_mean, dtype, device, seed)
    return tuple(x.reshape(B, H, d) for x in (q, k, v, g))


def random_state(B, H, d, device="cpu", seed=0, scale: Optional[float] = 1.0):
    """An fp32 recurrent state [B, H, d] ~ N(0, scale^2) (a carried-in prefix)."""
    gen = make_generator(device, seed)
    return torch.randn((B, H, d), generator=gen, device=device, dtype=torch.float32) * scale

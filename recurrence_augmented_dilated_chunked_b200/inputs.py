"""Seeded synthetic inputs for the RAT+ sequence mixer.

This module holds no arithmetic of the method: it only draws random tensors.
It is the one piece shared by the CUDA path's tests/benchmark and the fp64
oracle, so both sides see bit-identical inputs.

Recipe (one ``torch.Generator('cpu')`` per call, seeded): draw, in this order,
q, x_k, x_v and the gate logits z, each ``N(0, 1)`` in fp32 (z is then
``mean + std * N(0, 1)``); the gate is ``g = sigmoid(z)``, computed in fp32;
finally every tensor is cast once (round-to-nearest-even) to the run dtype.
The oracle reads the cast values, so input rounding is not charged as error.

The workloads are those of the RAT+ pages' model family: 1.5B-like
(d_model 2048, 16 heads of 128) and 7.6B-like (d_model 4096, 32 heads of 128)
layers, long-context T = 16K at D = 64 with a 128-token window, and decode
from 32K-token contexts.  There is no dataset: the pages' evaluation sets are
replaced by these Gaussian inputs.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    """One layer configuration of the hot path."""
    name: str
    dtype: str            # "f32" or "bf16"
    B: int
    T: int                # prefill tokens per sequence (0: decode-only)
    H: int
    Dh: int
    D: int
    W: int
    gate_mean: float
    gate_std: float
    dense_heads: tuple = field(default=())   # heads run dense (D = 1)
    decode_steps: int = 0
    decode_ctx: int = 0   # decode-only: tokens already in the cache

    @property
    def dense_mask(self):
        m = [0] * self.H
        for h in self.dense_heads:
            m[h] = 1
        return m


WORKLOADS = {
    w.name: w for w in [
        Workload("f32_small_T256_D4", "f32", B=1, T=256, H=2, Dh=64, D=4, W=0,
                 gate_mean=2.0, gate_std=1.0),
        Workload("bf16_1p5b_T4096_D16", "bf16", B=8, T=4096, H=16, Dh=128, D=16, W=0,
                 gate_mean=2.0, gate_std=1.5),
        Workload("bf16_long_T16384_D64_W128", "bf16", B=2, T=16384, H=16, Dh=128, D=64,
                 W=128, gate_mean=2.0, gate_std=1.5),
        Workload("bf16_decode_ctx32768_D64_W128", "bf16", B=64, T=0, H=16, Dh=128, D=64,
                 W=128, gate_mean=2.0, gate_std=1.5, decode_steps=256, decode_ctx=32768),
        Workload("bf16_hybrid_7p6b_T8192_D4", "bf16", B=4, T=8192, H=32, Dh=128, D=4, W=0,
                 gate_mean=1.0, gate_std=2.0, dense_heads=(0, 1), decode_steps=128),
    ]
}


def prefill_inputs(B, T, H, Dh, dtype="bf16", gate_mean=2.0, gate_std=1.0, seed=0):
    """Return (q, x_k, x_v, g), each [B, T, H, Dh] on the CPU in ``dtype``."""
    gen = torch.Generator("cpu").manual_seed(seed)
    shape = (B, T, H, Dh)
    q = torch.randn(shape, generator=gen, dtype=torch.float32)
    xk = torch.randn(shape, generator=gen, dtype=torch.float32)
    xv = torch.randn(shape, generator=gen, dtype=torch.float32)
    z = torch.randn(shape, generator=gen, dtype=torch.float32) * gate_std + gate_mean
    g = torch.sigmoid(z)
    dt = DTYPES[dtype]
    return q.to(dt), xk.to(dt), xv.to(dt), g.to(dt)


def decode_inputs(steps, B, H, Dh, dtype="bf16", gate_mean=2.0, gate_std=1.0, seed=1):
    """Per-step decode inputs (q, x_k, x_v, g), each [steps, B, H, Dh]."""
    gen = torch.Generator("cpu").manual_seed(seed)
    shape = (steps, B, H, Dh)
    q = torch.randn(shape, generator=gen, dtype=torch.float32)
    xk = torch.randn(shape, generator=gen, dtype=torch.float32)
    xv = torch.randn(shape, generator=gen, dtype=torch.float32)
    z = torch.randn(shape, generator=gen, dtype=torch.float32) * gate_std + gate_mean
    g = torch.sigmoid(z)
    dt = DTYPES[dtype]
    return q.to(dt), xk.to(dt), xv.to(dt), g.to(dt)


def decode_context(B, H, Dh, ctx, D, W, dense_mask=None, seed=2):
    """Synthetic already-prefilled decode context: every cached dilated row,
    every window-ring row and the fp32 recurrent state drawn from N(0, 1); a
    position held both as a dilated row and in the ring gets the one value.

    Returns (kd, vd, kw, vw, state): kd/vd are lists over heads of
    [B, ctx // D_h, Dh] bf16 tensors (row s = position s*D_h + D_h - 1);
    kw/vw are [B, H, W, Dh] bf16 in ring order (row r = the position
    p with p mod W == r among the last W); state is [2, B, H, Dh] fp32.
    """
    gen = torch.Generator("cpu").manual_seed(seed)
    kd, vd = [], []
    for h in range(H):
        Dd = 1 if (dense_mask is not None and dense_mask[h]) else D
        n = ctx // Dd
        kd.append(torch.randn((B, n, Dh), generator=gen).to(torch.bfloat16))
        vd.append(torch.randn((B, n, Dh), generator=gen).to(torch.bfloat16))
    Wr = max(W, 1)
    kw = torch.randn((B, H, Wr, Dh), generator=gen).to(torch.bfloat16)
    vw = torch.randn((B, H, Wr, Dh), generator=gen).to(torch.bfloat16)
    state = torch.randn((2, B, H, Dh), generator=gen, dtype=torch.float32)
    # a position kept in both places (a dilated one inside the last W) holds
    # one value, as it would after a prefill: the ring row repeats the slot
    if W > 0:
        for h in range(H):
            Dd = 1 if (dense_mask is not None and dense_mask[h]) else D
            for pos in range(max(0, ctx - W), ctx):
                if pos % Dd == Dd - 1:
                    kw[:, h, pos % W] = kd[h][:, pos // Dd]
                    vw[:, h, pos % W] = vd[h][:, pos // Dd]
    return kd, vd, kw, vw, state

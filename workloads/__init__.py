"""Seeded synthetic inputs for the retention hot path.

This module only draws random numbers and rounds them to the storage
dtype.  It holds none of the retention arithmetic: the CUDA library and
the CPU oracle each compute everything from these arrays on their own.

Shapes and distributions follow the five workloads used throughout the
repository (sizes of the RetNet summary page, "Key points": chunk b = 512,
head dimension 256, the 200M model's hidden size 1024):

  tiny       B=1, H=4,  n=256,  d=64,  fp32, q/k/v ~ N(0,1)/8,  chunk 64
  layer200m  B=8, H=4,  n=2048, d=256, bf16, q/k/v ~ N(0,1)/16, chunk 512 (and 64),
             gate G = X @ W_g, X [B*n, 1024] ~ N(0,1), W_g ~ N(0, 0.02)
  layer3b    B=4, H=10, n=2048, d=256, bf16, ~ N(0,1)/16, chunk 512, gate from
             X [B*n, 2560], W_g [2560, 2560]
  long7b     B=1, H=16, n=8192, d=256, bf16, ~ N(0,1)/16, chunk 512, emits state
  decode7b   H=16, d=256, state from an 8192-token random prefill, then 256 decode
             steps of bf16 q/k/v ~ N(0,1)/16, batch in {1, 8, 32, 128}

Draw order for a prefill workload with seed s (numpy default_rng(s)):
q, k, v (each float32 standard normal times the scale), then X, then W_g.
Values are rounded once to the workload dtype; both sides see the same bits.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = ["Workload", "WORKLOADS", "round_to_bf16", "make_prefill_inputs",
           "make_decode_inputs", "make_prefill_inputs_device", "make_msr_inputs", "normal"]


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    seqlen: int
    d: int
    dtype: str            # "f32" or "bf16"
    scale: float          # q, k, v ~ N(0,1) * scale
    chunk: int
    hidden: int = 0       # gate input width (0: no gate)
    seed: int = 0
    decode_steps: int = 0
    decode_batches: tuple = field(default_factory=tuple)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 256, 64, "f32", 1.0 / 8.0, 64, 0, 1000),
    "layer200m": Workload("layer200m", 8, 4, 2048, 256, "bf16", 1.0 / 16.0, 512, 1024, 1001),
    "layer3b": Workload("layer3b", 4, 10, 2048, 256, "bf16", 1.0 / 16.0, 512, 2560, 1002),
    "long7b": Workload("long7b", 1, 16, 8192, 256, "bf16", 1.0 / 16.0, 512, 0, 1003),
    "decode7b": Workload("decode7b", 1, 16, 8192, 256, "bf16", 1.0 / 16.0, 512, 0, 1004,
                         256, (1, 8, 32, 128)),
}


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even).

    Returns float32 values that are exactly representable in bf16.
    NaN/Inf are not expected in synthetic inputs and are not special-cased.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    return rounded.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 storage of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    raise ValueError(f"unknown dtype {dtype}")


def normal(rng: np.random.Generator, shape, scale: float, dtype: str) -> np.ndarray:
    return to_dtype(rng.standard_normal(shape, dtype=np.float32) * np.float32(scale), dtype)


def make_prefill_inputs(batch: int, heads: int, seqlen: int, d: int, dtype: str,
                        scale: float, seed: int, hidden: int = 0, dv: int | None = None):
    """q, k [B, n, H, d], v [B, n, H, dv] and (when hidden > 0) the gate G [B, n, H, dv].

    All arrays are float32 holding values representable in `dtype`.
    The gate is G = X @ W_g with X ~ N(0,1) of width `hidden` and
    W_g ~ N(0, 0.02) (std), computed in float32 and rounded to `dtype`.
    """
    dv = d if dv is None else dv
    rng = np.random.default_rng(seed)
    q = normal(rng, (batch, seqlen, heads, d), scale, dtype)
    k = normal(rng, (batch, seqlen, heads, d), scale, dtype)
    v = normal(rng, (batch, seqlen, heads, dv), scale, dtype)
    g = None
    if hidden:
        x = rng.standard_normal((batch * seqlen, hidden), dtype=np.float32)
        w = rng.standard_normal((hidden, heads * dv), dtype=np.float32) * np.float32(0.02)
        g = to_dtype((x @ w).reshape(batch, seqlen, heads, dv), dtype)
    return q, k, v, g


def make_msr_inputs(batch: int, seqlen: int, hidden: int, heads: int, d: int, seed: int):
    """Input and weights of the multi-scale retention layer, bf16 values.

    x [B, n, hidden] ~ N(0, 1); W_Q, W_K, W_V [H d, hidden] ~ N(0, s) with
    s = 1 / (16 sqrt(hidden)), so that the projected q, k, v have the
    prefill workloads' spread N(0, 1/16^2); W_G [H d, hidden] ~ N(0, 0.02),
    the gate weight of the layer workloads; W_O [hidden, H d] ~ N(0, 1/sqrt(H d)).
    Returns x, w_qkvg (the rows of W_Q, W_K, W_V, W_G stacked) and w_o.
    Draw order: x, W_Q, W_K, W_V, W_G, W_O.
    """
    rng = np.random.default_rng(seed)
    hd = heads * d
    x = normal(rng, (batch, seqlen, hidden), 1.0, "bf16")
    s = 1.0 / (16.0 * np.sqrt(hidden))
    wq, wk, wv = (normal(rng, (hd, hidden), s, "bf16") for _ in range(3))
    wg = normal(rng, (hd, hidden), 0.02, "bf16")
    wo = normal(rng, (hidden, hd), 1.0 / np.sqrt(hd), "bf16")
    return x, np.concatenate([wq, wk, wv, wg], axis=0), wo


def make_decode_inputs(batch: int, heads: int, steps: int, d: int, dtype: str,
                       scale: float, seed: int):
    """q, k, v [steps, batch, H, d] for a run of decode steps."""
    rng = np.random.default_rng(seed)
    q = normal(rng, (steps, batch, heads, d), scale, dtype)
    k = normal(rng, (steps, batch, heads, d), scale, dtype)
    v = normal(rng, (steps, batch, heads, d), scale, dtype)
    return q, k, v


def make_prefill_inputs_device(batch: int, heads: int, seqlen: int, d: int, scale: float,
                               seed: int, device, dtype=None):
    """q, k, v [B, n, H, d] drawn on `device` with torch's seeded generator.

    Same distribution as make_prefill_inputs (standard normal times `scale`,
    rounded to the storage dtype, bf16 by default), for workloads too large
    to draw on the host (the 8192-token prefills that seed decode states at
    batch 32 and 128).  The draw order is q, k, v.
    """
    import torch
    dtype = torch.bfloat16 if dtype is None else dtype
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    shape = (batch, seqlen, heads, d)
    out = []
    for _ in range(3):
        x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        out.append((x * scale).to(dtype))
        del x
    return tuple(out)

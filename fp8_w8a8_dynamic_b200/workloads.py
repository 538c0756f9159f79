"""Seeded synthetic inputs for the FP8_DYNAMIC Linear.

This module only draws random BF16 tensors and names shapes.  It holds none
of the method's arithmetic (no scales, no codes, no contraction), so the CUDA
path and the CPU oracle can both be fed from it without sharing anything else.

Shapes follow the language model described in the "MOSS-VL-Instruct-0708-FP8
architecture" article (model-architecture table: hidden 4096, 32 query heads,
8 KV heads, so head_dim 128 and k/v width 1024) and the "MOSS-VL quantization
README" FP8-Dynamic section (the seven projections q/k/v/o/gate/up/down of
each of the 36 layers without cross-attention).  The MLP width 12288 is an
assumption: the pages do not state it.

Value recipe (the pages give none; no dataset is used):
  X  ~ N(0, 1); for the "rowscale" kind every row is multiplied by
       r = exp(U(ln 0.1, ln 10)); then each entry independently, with
       probability 0.001, is multiplied by 50 (outliers).
  W  ~ N(0, std), std = 0.02 (times a per-layer jitter U(0.8, 1.2) for the
       252-Linear stack).
All draws are fp32 from ``torch.Generator(device)`` seeded per (seed, stream),
then rounded to BF16.  Parity tests copy the exact BF16 tensors to the host,
so no result depends on the generator being the same on CPU and GPU.
"""
import math
from dataclasses import dataclass

import torch

HIDDEN = 4096
N_HEADS = 32
N_KV_HEADS = 8
HEAD_DIM = HIDDEN // N_HEADS
KV_WIDTH = N_KV_HEADS * HEAD_DIM
INTERMEDIATE = 12288  # assumption, see module docstring
N_LAYERS = 48
CROSS_LAYERS = tuple(range(2, N_LAYERS, 4))
SELF_LAYERS = tuple(i for i in range(N_LAYERS) if i not in CROSS_LAYERS)


@dataclass(frozen=True)
class LinearShape:
    name: str
    K: int  # in_features
    N: int  # out_features


LAYER_LINEARS = (
    LinearShape("q_proj", HIDDEN, HIDDEN),
    LinearShape("k_proj", HIDDEN, KV_WIDTH),
    LinearShape("v_proj", HIDDEN, KV_WIDTH),
    LinearShape("o_proj", HIDDEN, HIDDEN),
    LinearShape("gate_proj", HIDDEN, INTERMEDIATE),
    LinearShape("up_proj", HIDDEN, INTERMEDIATE),
    LinearShape("down_proj", INTERMEDIATE, HIDDEN),
)
MLP_LINEARS = LAYER_LINEARS[4:]

# The same layer with the projections that read the same input packed into
# one Linear, as the README's packed modules do (qkv_proj, gate_up_proj):
# output channels concatenate, and so do their per-channel scales.
PACKED_LAYER_LINEARS = (
    LinearShape("qkv_proj", HIDDEN, HIDDEN + 2 * KV_WIDTH),
    LinearShape("o_proj", HIDDEN, HIDDEN),
    LinearShape("gate_up_proj", HIDDEN, 2 * INTERMEDIATE),
    LinearShape("down_proj", INTERMEDIATE, HIDDEN),
)


def generator(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    return g


def make_x(M: int, K: int, seed: int, stream: int = 0, kind: str = "normal",
           device="cpu") -> torch.Tensor:
    """Activations [M, K] BF16 (see module docstring for the recipe)."""
    g = generator(seed, stream, device)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    if kind == "rowscale":
        u = torch.rand(M, 1, generator=g, device=device, dtype=torch.float32)
        lo, hi = math.log(0.1), math.log(10.0)
        x = x * torch.exp(lo + u * (hi - lo))
    elif kind != "normal":
        raise ValueError(f"unknown activation kind {kind!r}")
    mask = torch.rand(M, K, generator=g, device=device, dtype=torch.float32) < 0.001
    x = torch.where(mask, x * 50.0, x)
    return x.to(torch.bfloat16)


def make_kv(T: int, H: int, D: int, seed: int, stream: int = 0, device="cpu") -> torch.Tensor:
    """Keys or values [T, H, D] BF16 for a cache whose groups run along the
    tokens: per (head, channel) column an offset ~ U(-2, 2) and a log-uniform
    spread in [0.1, 10] around it (so groups are asymmetric and of unequal
    width), N(0, 1) per token, and 0.1% outliers x50."""
    g = generator(seed, 20_000 + stream, device)
    x = torch.randn(T, H, D, generator=g, device=device, dtype=torch.float32)
    u = torch.rand(1, H, D, generator=g, device=device, dtype=torch.float32)
    off = torch.rand(1, H, D, generator=g, device=device, dtype=torch.float32) * 4.0 - 2.0
    lo, hi = math.log(0.1), math.log(10.0)
    x = x * torch.exp(lo + u * (hi - lo)) + off
    mask = torch.rand(T, H, D, generator=g, device=device, dtype=torch.float32) < 0.001
    x = torch.where(mask, x * 50.0, x)
    return x.to(torch.bfloat16)


def make_w(N: int, K: int, seed: int, stream: int = 0, std: float = 0.02,
           device="cpu") -> torch.Tensor:
    """Weights [N, K] BF16 in the Linear's (out_features, in_features) layout."""
    g = generator(seed, 10_000 + stream, device)
    w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * std
    return w.to(torch.bfloat16)


def layer_std_jitter(seed: int, n_layers: int) -> list:
    """Per-layer weight std multipliers u_l ~ U(0.8, 1.2), one per layer."""
    g = generator(seed, 99_999, "cpu")
    u = torch.rand(n_layers, generator=g, dtype=torch.float64)
    return [0.8 + 0.4 * float(v) for v in u]


# The five workloads, by index (the index is also the seed).
WORKLOADS = {
    0: dict(name="q_proj M=16", Ms=(16,), linears=(LAYER_LINEARS[0],), x_kind="normal"),
    1: dict(name="decode: 7 Linears of one layer at M in {1,4,8}", Ms=(1, 4, 8),
            linears=LAYER_LINEARS, x_kind="normal"),
    2: dict(name="prefill: 7 Linears of one layer at M=2048", Ms=(2048,),
            linears=LAYER_LINEARS, x_kind="rowscale"),
    3: dict(name="long-video prefill: gate/up/down at M=16384", Ms=(16384,),
            linears=MLP_LINEARS, x_kind="rowscale"),
    4: dict(name="252-Linear stack at M in {1,16,128,1024,8192}", Ms=(1, 16, 128, 1024, 8192),
            linears=LAYER_LINEARS, x_kind="normal", n_layers=len(SELF_LAYERS)),
}

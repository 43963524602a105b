"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws random numbers and rounds them to the storage types the
layer reads (bf16 bits, fp32).  It holds no step of the method itself, and it is
the one module that both the CPU oracle's tests and the CUDA path's tests / bench
take their inputs from, so both sides read identical bytes.

Workload shapes follow the pages' model (Gemma 4 26B-A4B: 30 MoE layers of 128
experts, hidden 2816, expert intermediate 704, top-8); the weights, routing
traces and prompts of that model are not available, so these draws stand in:

* expert weights ~ N(0, 0.02), activations ~ N(0, 1), both rounded to bf16 (RNE);
* router weights (the fp32 projection before the routing) ~ N(0, 0.02) in fp32,
  so that at hidden 2816 the projected logits are close to N(0, 1);
* router logits ~ N(0, 1) fp32 (uniform expert popularity);
* "biased": N(0, 1) plus a per-expert bias drawn once per layer from N(0, 1.5)
  (standard deviation 1.5), to skew popularity;
* "zipf": per layer a random expert permutation pi, and per token
  logit_e = -1.1 * log(rank_pi(e)) + Gumbel(0, 1); by the Gumbel-top-k property
  the top-k of these logits is a draw without replacement with probabilities
  proportional to Zipf(s = 1.1) weights.

Every draw comes from ``numpy.random.default_rng([seed, stream, ...])`` on the
host, or, for full-size weight stacks that live only on the GPU, from a seeded
``torch.Generator`` on that device (the bytes are read back wherever the oracle
needs them).
"""
from __future__ import annotations

import numpy as np

# stream ids, so that each tensor has its own sub-seed
S_W13, S_W2, S_X, S_LOGITS, S_BIAS, S_PERM, S_GUMBEL, S_ROUTER = 1, 2, 3, 4, 5, 6, 7, 8

WEIGHT_STD = 0.02


def bf16_bits(a) -> np.ndarray:
    """fp32 values -> bf16 bits, round to nearest even (NaN kept quiet)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    if nan.any():
        r = np.where(nan, ((u >> 16) | 0x40).astype(np.uint16), r)
    return r


def bf16_to_f32(bits) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), *[int(s) for s in stream]])


def normal_bf16(shape, std: float, seed: int, *stream: int) -> np.ndarray:
    g = _rng(seed, *stream)
    return bf16_bits(g.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def activations(T: int, H: int, seed: int = 0, layer: int = 0) -> np.ndarray:
    """x [T, H] as bf16 bits, N(0, 1)."""
    return normal_bf16((T, H), 1.0, seed, S_X, layer)


def expert_weights(E: int, H: int, I: int, seed: int = 0, layer: int = 0):
    """(w13 [E, 2I, H], w2 [E, H, I]) as bf16 bits, N(0, 0.02)."""
    w13 = normal_bf16((E, 2 * I, H), WEIGHT_STD, seed, S_W13, layer)
    w2 = normal_bf16((E, H, I), WEIGHT_STD, seed, S_W2, layer)
    return w13, w2


def router_weights(E: int, H: int, seed: int = 0, layer: int = 0) -> np.ndarray:
    """Router projection weights [E, H] fp32, N(0, 0.02)."""
    return _rng(seed, S_ROUTER, layer).standard_normal((E, H), dtype=np.float32) * np.float32(WEIGHT_STD)


def router_logits(T: int, E: int, kind: str = "normal", seed: int = 0, layer: int = 0,
                  step: int = 0) -> np.ndarray:
    """Router logits [T, E] fp32 for one layer (and one decode step)."""
    if kind == "normal":
        return _rng(seed, S_LOGITS, layer, step).standard_normal((T, E), dtype=np.float32)
    if kind == "biased":
        base = _rng(seed, S_LOGITS, layer, step).standard_normal((T, E), dtype=np.float32)
        bias = (_rng(seed, S_BIAS, layer).standard_normal(E, dtype=np.float32) * np.float32(1.5))
        return (base + bias[None, :]).astype(np.float32)
    if kind == "zipf":
        perm = _rng(seed, S_PERM, layer).permutation(E)
        rank = np.empty(E, np.int64)
        rank[perm] = np.arange(1, E + 1)
        base = (-1.1 * np.log(rank.astype(np.float64))).astype(np.float32)
        gum = _rng(seed, S_GUMBEL, layer, step).gumbel(size=(T, E)).astype(np.float32)
        return (base[None, :] + gum).astype(np.float32)
    raise ValueError(f"unknown logits kind {kind!r}")


# ---------------------------------------------------------------- device draws

def torch_normal_bf16(shape, std: float, seed: int, device, *stream: int):
    """N(0, std) drawn by a seeded torch generator on `device`, stored as bf16."""
    import torch

    g = torch.Generator(device=device)
    s = int(seed)
    for v in stream:
        s = (s * 1000003 + int(v) + 1) % (2**62)
    g.manual_seed(s)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    # draw in fp32 slices so the host never holds the tensor and device memory stays bounded
    flat = out.view(-1)
    step = 1 << 26
    for i in range(0, flat.numel(), step):
        n = min(step, flat.numel() - i)
        flat[i:i + n] = (torch.randn(n, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)
    return out


def torch_expert_weights(E: int, H: int, I: int, seed: int, layer: int, device):
    """(w13 [E, 2I, H], w2 [E, H, I]) bf16 tensors on `device`, N(0, 0.02)."""
    w13 = torch_normal_bf16((E, 2 * I, H), WEIGHT_STD, seed, device, S_W13, layer)
    w2 = torch_normal_bf16((E, H, I), WEIGHT_STD, seed, device, S_W2, layer)
    return w13, w2


# -------------------------------------------------------------- the workloads

# name -> (E, H, I, k, T list, weight format, logits kind)
CONFIGS = {
    "tiny": dict(E=8, H=256, I=128, k=2, T=[16], fmt="bf16", logits="normal"),
    "decode-bf16": dict(E=128, H=2816, I=704, k=8, T=[1, 8, 64], fmt="bf16", logits="normal"),
    "decode-int8": dict(E=128, H=2816, I=704, k=8, T=[1, 8, 64], fmt="int8", logits="biased"),
    "int4": dict(E=128, H=2816, I=704, k=8, T=[1024, 64], fmt="int4", logits="normal"),
    "stack30": dict(E=128, H=2816, I=704, k=8, T=[1, 8, 64], fmt="int4", logits="zipf", L=30,
                    slots_per_layer=18, refresh_every=8, steps=256),
}

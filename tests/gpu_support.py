"""Helpers shared by the GPU parity tests: build the same layer on both sides
from the same seeded bf16 weights -- the oracle quantises and packs its own
blobs on the host, the CUDA path quantises and packs on the device -- and the
error measure the tests use."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synthetic as syn

# FFN tolerance: max|gpu - oracle| / max|oracle| (fp32 accumulation with bf16
# rounding of the intermediate h on the GPU, fp64 in the oracle).
FFN_TOL = 1e-2


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    return float(np.abs(gpu - ref).max() / (den if den > 0 else 1.0))


def bf16_dev_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def oracle_blob(fmt: int, w13_bits: np.ndarray, w2_bits: np.ndarray, H: int, I: int) -> np.ndarray:
    """One expert's blob built by the oracle's own quantiser and packer."""
    if fmt == oracle.BF16:
        return oracle.pack_expert(fmt, H, I, w13_bits, None, w2_bits, None)
    if fmt == oracle.INT8:
        q13, s13 = oracle.quantize_int8(w13_bits)
        q2, s2 = oracle.quantize_int8(w2_bits)
    else:
        q13, s13 = oracle.quantize_int4(w13_bits)
        q2, s2 = oracle.quantize_int4(w2_bits)
    return oracle.pack_expert(fmt, H, I, q13, s13, q2, s2)


def oracle_layer_for(fmt: int, w13_bits: np.ndarray, w2_bits: np.ndarray, experts=None) -> oracle.Layer:
    """Oracle view of a layer.  With `experts`, only those experts get blobs: they
    are placed in a compact pool behind a slot table (home is never read)."""
    E, I2, H = w13_bits.shape
    I = I2 // 2
    eb = oracle.expert_bytes(fmt, H, I)
    if experts is None:
        home = np.concatenate([oracle_blob(fmt, w13_bits[e], w2_bits[e], H, I) for e in range(E)])
        return oracle.Layer(fmt, E, H, I, home)
    experts = sorted(set(int(e) for e in experts))
    slot = np.full(E, -1, np.int32)
    pool = np.zeros(max(len(experts), 1) * eb, np.uint8)
    for i, e in enumerate(experts):
        slot[e] = i
        pool[i * eb:(i + 1) * eb] = oracle_blob(fmt, w13_bits[e], w2_bits[e], H, I)
    return oracle.Layer(fmt, E, H, I, np.zeros(eb, np.uint8), pool=pool, slot_table=slot)


def device_weights_from_host(w13_bits: np.ndarray, w2_bits: np.ndarray, dev="cuda"):
    w13 = torch.from_numpy(w13_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    w2 = torch.from_numpy(w2_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    return w13, w2


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

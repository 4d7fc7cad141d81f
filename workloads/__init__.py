"""Seeded synthetic inputs shared by the tests, the benchmark and smoke().

This module draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the fp64 oracle and the CUDA library can be fed
from it without sharing any of the method.

Recipe (shapes from ``MiMoV2FlashConfig``: 64 query heads, 4 key/value heads,
``head_dim=192``, ``v_head_dim=128``, ``sliding_window=129``):

* q / k / v: ``torch.randn`` float32 from a seeded generator, rounded to
  bfloat16 (round-to-nearest-even) -- values ~N(0, 1).
* sink logits: float32 ~N(0, 1), one per query head (per layer for stacks).
* sequence lengths: ``numpy.random.default_rng(seed).integers(lo, hi + 1, n)``.
* decode caches: slots holding tokens that exist are ~N(0, 1); slots past a
  sequence's length are filled with NaN ("poison") unless ``poison=False`` so
  that any read of an invalid slot shows up in the output.
* FP8 decode caches: the same N(0, 1) draws divided by a fixed per-KV-head
  scale (K: (8 + g) / 448, V: (6 + 2 g) / 448, so about +-8 sigma spans the
  e4m3 range), clamped to +-448 and rounded to e4m3 by torch's float8_e4m3fn
  cast; poison slots hold the NaN code 0x7F.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

HQ, HKV, DQK, DV, SWA_WINDOW = 64, 4, 192, 128, 129


def lengths_uniform(seed, n, lo, hi):
    """n integer lengths ~Uniform[lo, hi] (inclusive) from ``default_rng(seed)``."""
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, n)]


def cu_seqlens_of(lengths):
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape, gen, device="cpu"):
    return torch.randn(shape, generator=gen, dtype=torch.float32, device=device).to(torch.bfloat16)


@dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    sinks: torch.Tensor | None
    cu_seqlens: torch.Tensor
    lengths: list = field(default_factory=list)

    @property
    def total(self):
        return int(self.q.shape[0])


def prefill_inputs(lengths, hq=HQ, hkv=HKV, dqk=DQK, dv=DV, seed=0,
                   sinks=True, device="cpu"):
    """Packed varlen prefill inputs: q [Nt,Hq,Dqk], k [Nt,Hkv,Dqk], v [Nt,Hkv,Dv]."""
    nt = int(sum(lengths))
    g = _gen(seed, device)
    q = randn_bf16((nt, hq, dqk), g, device)
    k = randn_bf16((nt, hkv, dqk), g, device)
    v = randn_bf16((nt, hkv, dv), g, device)
    s = torch.randn(hq, generator=g, dtype=torch.float32, device=device) if sinks else None
    return PrefillInputs(q, k, v, s, cu_seqlens_of(lengths).to(device), list(lengths))


def stack_sinks(num_layers, hq=HQ, seed=0, device="cpu"):
    """Per-layer, per-head sink logits [num_layers, Hq] ~N(0,1)."""
    g = _gen(seed + 7919, device)
    return torch.randn((num_layers, hq), generator=g, dtype=torch.float32, device=device)


@dataclass
class DecodeInputs:
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    seqlens: torch.Tensor
    sinks: torch.Tensor | None
    window: int
    capacity: int


def decode_inputs(seqlens, capacity, window, hq=HQ, hkv=HKV, dqk=DQK, dv=DV,
                  seed=0, sinks=True, poison=True, device="cpu"):
    """One decode step: q [B,Hq,Dqk], caches [B,C,Hkv,D], seqlens [B] int32.

    ``seqlens[b]`` counts the current token (already written to the cache).
    For a ring cache (``window > 0`` and ``capacity == window``) every slot
    below ``min(L, C)`` holds a token; for a linear cache slots ``< L`` do.
    """
    B = len(seqlens)
    g = _gen(seed, device)
    q = randn_bf16((B, hq, dqk), g, device)
    k = torch.empty((B, capacity, hkv, dqk), dtype=torch.bfloat16, device=device)
    v = torch.empty((B, capacity, hkv, dv), dtype=torch.bfloat16, device=device)
    for b, L in enumerate(seqlens):
        n = min(int(L), capacity)
        k[b, :n] = randn_bf16((n, hkv, dqk), g, device)
        v[b, :n] = randn_bf16((n, hkv, dv), g, device)
        fill = float("nan") if poison else 0.0
        if n < capacity:
            k[b, n:] = fill
            v[b, n:] = fill
    s = torch.randn(hq, generator=g, dtype=torch.float32, device=device) if sinks else None
    sl = torch.tensor([int(L) for L in seqlens], dtype=torch.int32, device=device)
    return DecodeInputs(q, k, v, sl, s, window, capacity)


@dataclass
class DecodeInputsFp8:
    q: torch.Tensor
    k_codes: torch.Tensor    # uint8 e4m3 codes [B, C, Hkv, Dqk]
    v_codes: torch.Tensor    # uint8 e4m3 codes [B, C, Hkv, Dv]
    k_scale: torch.Tensor    # [Hkv] fp32
    v_scale_kv: torch.Tensor  # [Hkv] fp32
    seqlens: torch.Tensor
    sinks: torch.Tensor | None
    window: int
    capacity: int


def fp8_kv_scales(hkv=HKV, device="cpu"):
    """Fixed per-KV-head cache scales (K, V) used by the FP8 decode workloads."""
    k = torch.tensor([(8.0 + g) / 448.0 for g in range(hkv)], dtype=torch.float32, device=device)
    v = torch.tensor([(6.0 + 2.0 * g) / 448.0 for g in range(hkv)], dtype=torch.float32, device=device)
    return k, v


def _e4m3_codes(x, scale):
    y = (x / scale.view(1, -1, 1)).clamp_(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8)


def decode_inputs_fp8(seqlens, capacity, window, hq=HQ, hkv=HKV, dqk=DQK, dv=DV,
                      seed=0, sinks=True, poison=True, device="cpu"):
    """One decode step over e4m3 caches: q [B,Hq,Dqk] bf16, uint8 codes, per-head scales."""
    B = len(seqlens)
    g = _gen(seed, device)
    q = randn_bf16((B, hq, dqk), g, device)
    ks, vs = fp8_kv_scales(hkv, device)
    k = torch.empty((B, capacity, hkv, dqk), dtype=torch.uint8, device=device)
    v = torch.empty((B, capacity, hkv, dv), dtype=torch.uint8, device=device)
    for b, L in enumerate(seqlens):
        n = min(int(L), capacity)
        k[b, :n] = _e4m3_codes(torch.randn((n, hkv, dqk), generator=g, dtype=torch.float32,
                                           device=device), ks)
        v[b, :n] = _e4m3_codes(torch.randn((n, hkv, dv), generator=g, dtype=torch.float32,
                                           device=device), vs)
        if n < capacity:
            k[b, n:] = 0x7F if poison else 0
            v[b, n:] = 0x7F if poison else 0
    s = torch.randn(hq, generator=g, dtype=torch.float32, device=device) if sinks else None
    sl = torch.tensor([int(L) for L in seqlens], dtype=torch.int32, device=device)
    return DecodeInputsFp8(q, k, v, ks, vs, sl, s, window, capacity)


# The five workloads, by what they are.
TINY_SWA = dict(name="tiny SWA prefill T=512 Hq=16 Hkv=1 W=129 (fp32 out)",
                lengths=[512], hq=16, hkv=1, window=129, out_dtype="f32")
SWA_32K = dict(name="SWA prefill T=32768 Hq=64 Hkv=4 W=129",
               lengths=[32768], hq=HQ, hkv=HKV, window=SWA_WINDOW, out_dtype="bf16")
GA_32K = dict(name="global prefill T=32768 Hq=64 Hkv=4",
              lengths=[32768], hq=HQ, hkv=HKV, window=0, out_dtype="bf16")


def decode_b64_lengths(seed=0):
    """Global-layer decode lengths ~Uniform[1024, 262144] for 64 sequences."""
    return lengths_uniform(seed, 64, 1024, 262144)


DECODE_GA_CAPACITY = 262144


def varlen_stack_lengths(seed=0):
    """16 packed sequences, lengths ~Uniform[512, 8192]."""
    return lengths_uniform(seed, 16, 512, 8192)


#: 5:1 hybrid stack: layers 0-4 sliding window (129), layer 5 global.
STACK_WINDOWS = [SWA_WINDOW] * 5 + [0]

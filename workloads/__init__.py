"""Seeded synthetic attention workloads.

This module only draws random numbers and describes shapes. It holds none of
the attention arithmetic, so that the CPU oracle and the CUDA path can both be
fed from it without sharing any of the method's code.

The five workloads take the shapes of the experiments the FlashAttention pages
report ("FlashAttention (UR)", section "Experimental results": BERT-large at
length 512, GPT-2 at length 1K, Long-Range Arena at 1K-4K) plus a tiny
correctness case and a long-context single-batch case. No model, weights or
dataset is involved: every tensor is i.i.d. N(0, 1) rounded to bfloat16.

Recipe (fixed, so any run can be reproduced):
  * generator: ``torch.Generator('cpu').manual_seed(seed)``;
  * draw order: Q, then K, then V, each ``torch.randn`` in fp32 of shape
    ``[B, H, N, d]`` (K and V: ``[B, H_kv, N, d]`` for grouped-query shapes),
    then ``.to(torch.bfloat16)`` (round to nearest even);
  * ``q_mult`` (long-range case): Q is multiplied by 4 after rounding, which is
    exact in bf16 because 4 is a power of two;
  * key padding (BERT-shaped case): after V,
    ``kv_len = torch.randint(kv_lo, kv_hi + 1, (B,))`` from the same generator;
  * default seed: the workload's index (1..5).

Beyond the five square workloads: `DECODE_WORKLOADS` (one query row per head
against a long key/value cache, for the split-KV path) with `make_qkv` (separate
query and key counts); `make_bwd_inputs` (Q, K, V, then the output gradient dO,
for the backward); `make_fp8_inputs` (the same N(0,1) draws quantized per tensor
to e4m3 by torch's float8 conversion, for the e4m3 forward). Each keeps the
draw order Q, K, V (then dO), then kv_len.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    H: int
    N: int
    d: int
    causal: bool
    q_mult: float = 1.0
    kv_len_range: Optional[tuple] = None  # (lo, hi) inclusive, or None
    H_kv: Optional[int] = None            # K/V heads (grouped/multi-query); None = H

    @property
    def kv_heads(self) -> int:
        return self.H if self.H_kv is None else self.H_kv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def units(self) -> int:
        """Query tiles of 128 rows: the independent work units."""
        return self.B * self.H * ((self.N + 127) // 128)

    def flops(self) -> float:
        """Counted FLOPs of the metric: 4*B*H*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "B": self.B, "H": self.H, "H_kv": self.kv_heads, "N": self.N, "d": self.d,
            "causal": self.causal,
            "mask": ("causal" if self.causal else
                     ("key_padding" if self.kv_len_range else "none")),
            "q_mult": self.q_mult,
            "scale": self.scale,
        }


WORKLOADS = [
    Workload("tiny_noncausal_B1_H2_N256_d64", 1, 1, 2, 256, 64, False),
    Workload("bert_large_keypad_B16_H16_N512_d64", 2, 16, 16, 512, 64, False,
             kv_len_range=(256, 512)),
    Workload("gpt2_causal_B8_H12_N1024_d64", 3, 8, 12, 1024, 64, True),
    Workload("long_range_causal_qx4_B2_H16_N4096_d128", 4, 2, 16, 4096, 128, True,
             q_mult=4.0),
    Workload("long_context_causal_B1_H32_N16384_d128", 5, 1, 32, 16384, 128, True),
]

BY_NAME = {w.name: w for w in WORKLOADS}
BY_INDEX = {w.index: w for w in WORKLOADS}


def get(key) -> Workload:
    if isinstance(key, int):
        return BY_INDEX[key]
    if isinstance(key, str) and key.isdigit():
        return BY_INDEX[int(key)]
    return BY_NAME[key]


def make_inputs(w: Workload, seed: Optional[int] = None):
    """Return (q, k, v, kv_len) on the CPU; q bf16 [B,H,N,d], k/v bf16
    [B,H_kv,N,d] (H_kv = H unless grouped), kv_len int32 [B] or None."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.index if seed is None else seed)
    shape = (w.B, w.H, w.N, w.d)
    kv_shape = (w.B, w.kv_heads, w.N, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(kv_shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(kv_shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    if w.q_mult != 1.0:
        q = q * w.q_mult
    kv_len = None
    if w.kv_len_range is not None:
        lo, hi = w.kv_len_range
        kv_len = torch.randint(lo, hi + 1, (w.B,), generator=g).to(torch.int32)
    return q, k, v, kv_len


def make_custom(B, H, N, d, seed, q_mult=1.0, kv_len_range=None):
    """Same recipe for an arbitrary shape (ragged-tail and edge-case tests)."""
    w = Workload(f"custom_B{B}_H{H}_N{N}_d{d}", 0, B, H, N, d, False, q_mult,
                 kv_len_range)
    return make_inputs(w, seed=seed)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Few query rows against a long key/value cache (split-KV path): q
    [B, H, Nq, d], k, v [B, H_kv, Nk, d], query row i at key position
    i + Nk - Nq."""
    name: str
    B: int
    H: int
    H_kv: int
    Nq: int
    Nk: int
    d: int
    causal: bool = True
    seed: int = 11

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """4*B*H*Nq*Nk*d (every query row sees every key when Nq == 1)."""
        return 4.0 * self.B * self.H * self.Nq * self.Nk * self.d

    def algorithmic_bytes(self) -> int:
        """K and V read once, Q read once, O and lse written once."""
        kv = 2 * self.B * self.H_kv * self.Nk * self.d * 2
        qo = 2 * self.B * self.H * self.Nq * self.d * 2
        return kv + qo + self.B * self.H * self.Nq * 4

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "H_kv": self.H_kv,
                "Nq": self.Nq, "Nk": self.Nk, "d": self.d, "causal": self.causal,
                "scale": self.scale}


# Decoding one token per sequence against an 8K-token cache with grouped
# K/V heads (4 query heads per K/V head), the inference setting the pages'
# specialised kernels target ("FlashAttention (UR)", "Specialised solutions").
DECODE_WORKLOADS = [
    DecodeWorkload("decode_gqa_B16_H32_Hkv8_Nq1_Nk8192_d128", 16, 32, 8, 1, 8192, 128),
    # one sequence against a 128K-token cache: too few head groups to fill the
    # SMs, so the keys are split into ranges and merged
    DecodeWorkload("decode_gqa_B1_H32_Hkv8_Nq1_Nk131072_d128", 1, 32, 8, 1, 131072, 128,
                   seed=12),
]
DECODE_BY_NAME = {w.name: w for w in DECODE_WORKLOADS}


def make_qkv(B, H, H_kv, Nq, Nk, d, seed, kv_len_range=None):
    """Same recipe with separate query and key counts: q [B,H,Nq,d], then k
    and v [B,H_kv,Nk,d], then kv_len (if a range is given)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((B, H_kv, Nk, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((B, H_kv, Nk, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    kv_len = None
    if kv_len_range is not None:
        lo, hi = kv_len_range
        kv_len = torch.randint(lo, hi + 1, (B,), generator=g).to(torch.int32)
    return q, k, v, kv_len


def make_bwd_inputs(B, H, H_kv, N, d, seed, kv_len_range=None, q_mult=1.0):
    """Inputs of a backward pass: q [B,H,N,d], k, v [B,H_kv,N,d], then the
    output gradient dO [B,H,N,d] (N(0,1), rounded to bf16), then kv_len."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, H, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((B, H_kv, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((B, H_kv, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    do = torch.randn((B, H, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    if q_mult != 1.0:
        q = q * q_mult
    kv_len = None
    if kv_len_range is not None:
        lo, hi = kv_len_range
        kv_len = torch.randint(lo, hi + 1, (B,), generator=g).to(torch.int32)
    return q, k, v, do, kv_len


def make_fp8_inputs(B, H, H_kv, N, d, seed, kv_len_range=None, Nk=None):
    """e4m3 inputs: the same draws as make_inputs (Q, then K, then V, N(0,1)
    fp32), each divided by its descale amax / 448 and rounded to e4m3 by
    torch's float8_e4m3fn conversion (round to nearest even, no saturation
    needed). q has N rows, k and v Nk (default N) keys. Returns (q8, k8, v8,
    (q_descale, k_descale, v_descale), kv_len)."""
    Nk = N if Nk is None else Nk
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    xs = [torch.randn(shape, generator=g, dtype=torch.float32)
          for shape in ((B, H, N, d), (B, H_kv, Nk, d), (B, H_kv, Nk, d))]
    kv_len = None
    if kv_len_range is not None:
        lo, hi = kv_len_range
        kv_len = torch.randint(lo, hi + 1, (B,), generator=g).to(torch.int32)
    out, scales = [], []
    for x in xs:
        amax = float(x.abs().max()) if x.numel() else 1.0
        sc = (amax / 448.0) if amax > 0 else 1.0
        out.append((x / sc).to(torch.float8_e4m3fn))
        scales.append(sc)
    return out[0], out[1], out[2], tuple(scales), kv_len


def sample_rows(N: int, seed: int, n_random: int = 256, edge: int = 128):
    """Row indices for sampled checks at full size: the first and last `edge`
    rows plus `n_random` seeded random rows, sorted and unique."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    rows = set(range(min(edge, N))) | set(range(max(0, N - edge), N))
    if N > 0:
        rows |= set(torch.randint(0, N, (n_random,), generator=g).tolist())
    return sorted(rows)

"""FP8 (e4m3) inputs for the CPU oracle (test infrastructure only).

The FP8 forward takes Q, K, V as 8-bit e4m3 codes with one fp32 descale
factor per tensor and computes the attention of the dequantized tensors
descale * decode(code) -- the FlashAttention-3 direction of lower-precision
inputs ("FlashAttention (UR)", section "FlashAttention-3"). The pages fix no
format details; e4m3 here is the OCP 8-bit float with 1 sign bit, 4 exponent
bits (bias 7), 3 mantissa bits, subnormals, no infinities, and the single NaN
pattern S.1111.111 (largest finite 448).

`decode_e4m3` writes that definition out; `attention_fp8` dequantizes in fp64
(exact: every e4m3 value times an fp32 descale is an fp64 number) and calls
the pinned fp64 oracle.
"""
from __future__ import annotations

import numpy as np

import oracle


def decode_e4m3(codes) -> np.ndarray:
    """float64 values of e4m3 codes (uint8 array-like)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    subnormal = np.ldexp(m / 8.0, -6)
    val = sign * np.where(e == 0, subnormal, normal)
    return np.where((e == 15) & ((c & 7) == 7), np.nan, val)


def _codes(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype != torch.uint8:
                x = x.view(torch.uint8)
            return x.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.uint8)


def attention_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale, causal=False,
                  kv_len=None, rows=None, nthreads=0, lib=None):
    """Exact fp64 attention of the dequantized e4m3 tensors (q8 [B,H,N,d], k8 and
    v8 [B,H_kv,N,d], as uint8 codes or torch float8_e4m3fn tensors)."""
    q = decode_e4m3(_codes(q8)) * float(q_descale)
    k = decode_e4m3(_codes(k8)) * float(k_descale)
    v = decode_e4m3(_codes(v8)) * float(v_descale)
    return oracle.attention(q, k, v, scale, causal=causal, kv_len=kv_len, rows=rows,
                            nthreads=nthreads, lib=lib)

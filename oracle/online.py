"""Blockwise online-softmax attention in fp64 numpy (test infrastructure only).

A second, independent evaluation order of the same attention, written from
"FlashAttention (UR)", section "Online softmax": the keys are visited one block
at a time, and two running per-row quantities -- the largest score seen so far
(m) and the sum of exponentials relative to it (l) -- are updated as each block
arrives. Whenever m grows, the partial sum and the partial output are scaled by
exp(m_old - m_new) so that all terms stay relative to the current maximum. The
page states that this reaches the exact softmax without ever holding a full
score row; the tests check that claim against the two-pass oracle.

Masking and readings are the oracle's: additive -inf; causal key j visible iff
j <= i; keys j >= kv_len[b] hidden; a row with no visible key gives O = 0 and
lse = -inf.
"""
from __future__ import annotations

import numpy as np


def attention_online(q, k, v, scale, causal=False, kv_len=None, block=64):
    """q, k, v: float64 arrays [B, H, N, d]. Returns (o, lse) like the oracle."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, N, d = q.shape
    if block < 1:
        raise ValueError("block must be >= 1")
    o = np.zeros((B, H, N, d))
    lse = np.full((B, H, N), -np.inf)
    rows = np.arange(N)
    for b in range(B):
        lim = N if kv_len is None else int(min(max(int(kv_len[b]), 0), N))
        for h in range(H):
            m = np.full(N, -np.inf)      # running row max
            l = np.zeros(N)              # running sum of exp(s - m)
            acc = np.zeros((N, d))       # running sum of exp(s - m) * v
            for j0 in range(0, N, block):
                j1 = min(j0 + block, N)
                cols = np.arange(j0, j1)
                s = scale * (q[b, h] @ k[b, h, j0:j1].T)       # [N, blk]
                hidden = cols[None, :] >= lim
                if causal:
                    hidden = hidden | (cols[None, :] > rows[:, None])
                s = np.where(hidden, -np.inf, s)
                m_blk = s.max(axis=1)
                m_new = np.maximum(m, m_blk)
                live = m_new > -np.inf
                # factor that re-expresses old partial sums relative to m_new
                alpha = np.where(live & (m > -np.inf),
                                 np.exp(np.where(live, m - m_new, 0.0)), 0.0)
                p = np.where(live[:, None],
                             np.exp(s - np.where(live, m_new, 0.0)[:, None]), 0.0)
                l = alpha * l + p.sum(axis=1)
                acc = alpha[:, None] * acc + p @ v[b, h, j0:j1]
                m = np.where(live, m_new, m)
            seen = l > 0
            o[b, h] = np.where(seen[:, None], acc / np.where(seen, l, 1.0)[:, None], 0.0)
            lse[b, h] = np.where(seen, m + np.log(np.where(seen, l, 1.0)), -np.inf)
    return o, lse

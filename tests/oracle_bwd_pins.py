"""Pins for the backward part of the CPU oracle (oracle.attention_bwd).

The pages state no backward algorithm; the oracle's gradients are the exact
derivatives of the forward definition ("FlashAttention (UR)", section
"Problem of standard attention"). Each pin checks them against something
that does not share their arithmetic:

  * central finite differences of the (separately pinned) forward oracle;
  * torch autograd through torch's fp64 scaled_dot_product_attention;
  * two invariants of the definition: a shift common to all keys leaves
    every softmax row unchanged, so sum_j dK_j = 0; rows of P sum to one, so
    sum_j dV_j = sum_i dO_i over the rows that see a key;
  * dO = 0 gives zero gradients; bf16 and fp64 inputs of equal value agree.

Each function takes the oracle library handle (so the mutation test can run
the battery against planted mistakes) and raises AssertionError on a mismatch.
"""
from __future__ import annotations

import numpy as np

import oracle


def _bwd(lib, q, k, v, do, scale, causal=False, kv_len=None):
    return oracle.attention_bwd(q, k, v, do, scale, causal=causal, kv_len=kv_len, nthreads=1,
                                lib=lib)


def _loss(lib, q, k, v, g, scale, causal, kv_len):
    o, _ = oracle.attention(q, k, v, scale, causal=causal, kv_len=kv_len, nthreads=1, lib=lib)
    return float(np.sum(o * g))


def pin_bwd_finite_differences(lib):
    rng = np.random.default_rng(11)
    eps = 1e-5
    for Hkv, causal, kv_len in ((2, False, None), (1, True, None), (1, False, [4])):
        B, H, N, d, scale = 1, 2, 6, 3, 0.7
        q = rng.standard_normal((B, H, N, d))
        k = rng.standard_normal((B, Hkv, N, d))
        v = rng.standard_normal((B, Hkv, N, d))
        g = rng.standard_normal((B, H, N, d))
        grads = _bwd(lib, q, k, v, g, scale, causal, kv_len)
        for x, gx in zip((q, k, v), grads):
            for idx in np.ndindex(x.shape):
                x0 = x[idx]
                x[idx] = x0 + eps
                lp = _loss(lib, q, k, v, g, scale, causal, kv_len)
                x[idx] = x0 - eps
                lm = _loss(lib, q, k, v, g, scale, causal, kv_len)
                x[idx] = x0
                fd = (lp - lm) / (2 * eps)
                assert abs(gx[idx] - fd) <= 1e-7 * (1 + abs(fd)), (Hkv, causal, kv_len, idx,
                                                                     gx[idx], fd)


def pin_bwd_torch_autograd(lib):
    import torch
    rng = np.random.default_rng(12)
    for causal, kv_len in ((False, None), (True, None), (False, [5, 9])):
        B, H, Hkv, N, d, scale = 2, 4, 2, 9, 5, 0.45
        q = rng.standard_normal((B, H, N, d))
        k = rng.standard_normal((B, Hkv, N, d))
        v = rng.standard_normal((B, Hkv, N, d))
        g = rng.standard_normal((B, H, N, d))
        dq, dk, dv = _bwd(lib, q, k, v, g, scale, causal, kv_len)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        rep = H // Hkv
        kk = tk.repeat_interleave(rep, dim=1)
        vv = tv.repeat_interleave(rep, dim=1)
        mask = torch.ones(B, 1, N, N, dtype=torch.bool)
        if kv_len is not None:
            for b in range(B):
                mask[b, :, :, kv_len[b]:] = False
        if causal:
            mask &= torch.ones(N, N, dtype=torch.bool).tril()
        o = torch.nn.functional.scaled_dot_product_attention(tq, kk, vv, attn_mask=mask,
                                                             scale=scale)
        o.backward(torch.tensor(g))
        for a, t in ((dq, tq), (dk, tk), (dv, tv)):
            assert np.abs(a - t.grad.numpy()).max() <= 1e-11, (causal, kv_len)


def pin_bwd_invariants(lib):
    rng = np.random.default_rng(13)
    for causal, kv_len, Hkv in ((False, None, 3), (True, None, 1), (False, [7, 20], 3)):
        B, H, N, d, scale = 2, 3, 20, 6, 0.4
        q = rng.standard_normal((B, H, N, d))
        k = rng.standard_normal((B, Hkv, N, d))
        v = rng.standard_normal((B, Hkv, N, d))
        g = rng.standard_normal((B, H, N, d))
        dq, dk, dv = _bwd(lib, q, k, v, g, scale, causal, kv_len)
        # a shift common to all keys changes no softmax row
        assert np.abs(dk.sum(axis=2)).max() <= 1e-11
        # rows of P sum to one: sum over keys of dV = sum over query rows of dO
        rep = H // Hkv
        for b in range(B):
            for hk in range(Hkv):
                rows = g[b, hk * rep:(hk + 1) * rep].sum(axis=(0, 1))
                assert np.abs(dv[b, hk].sum(axis=0) - rows).max() <= 1e-11
        # hidden keys get no gradient
        if kv_len is not None:
            for b in range(B):
                assert np.all(dk[b, :, kv_len[b]:] == 0) and np.all(dv[b, :, kv_len[b]:] == 0)


def pin_bwd_zero_output_gradient(lib):
    rng = np.random.default_rng(14)
    q, k, v = (rng.standard_normal((1, 2, 8, 4)) for _ in range(3))
    for a in _bwd(lib, q, k, v, np.zeros_like(q), 0.5, True):
        assert np.all(a == 0)


def pin_bwd_bf16_inputs_equal_f64(lib):
    import torch
    g = torch.Generator().manual_seed(15)
    xs = [torch.randn(1, 4, 12, 8, generator=g).to(torch.bfloat16) for _ in range(2)]
    kv = [torch.randn(1, 2, 12, 8, generator=g).to(torch.bfloat16) for _ in range(2)]
    q, do = xs
    k, v = kv
    a = _bwd(lib, q, k, v, do, 0.35, True, [9])
    b = _bwd(lib, *(x.double() for x in (q, k, v, do)), 0.35, True, [9])
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def pin_bwd_dq_rows_equal_full(lib):
    """The row-subset driver gives exactly the full backward's dQ rows."""
    import torch
    g = torch.Generator().manual_seed(16)
    q, do = (torch.randn(2, 4, 33, 8, generator=g).to(torch.bfloat16) for _ in range(2))
    k, v = (torch.randn(2, 2, 33, 8, generator=g).to(torch.bfloat16) for _ in range(2))
    rows = [0, 5, 17, 32]
    for causal, kv_len in ((True, None), (False, [20, 33])):
        full, _, _ = _bwd(lib, q, k, v, do, 0.4, causal, kv_len)
        part = oracle.attention_bwd_dq_rows(q, k, v, do, 0.4, rows, causal=causal,
                                            kv_len=kv_len, nthreads=1, lib=lib)
        assert np.array_equal(part, full[:, :, rows]), (causal, kv_len)


def pin_bwd_kv_rows_equal_full(lib):
    """The key-row driver gives the full backward's dK and dV rows (to fp64
    rounding: it sums the query rows in another order), with grouped heads,
    causal and padding masks, and keys no row sees (all-zero rows)."""
    import torch
    g = torch.Generator().manual_seed(17)
    q, do = (torch.randn(2, 4, 40, 8, generator=g).to(torch.bfloat16) for _ in range(2))
    k, v = (torch.randn(2, 2, 40, 8, generator=g).to(torch.bfloat16) for _ in range(2))
    rows = [0, 1, 13, 25, 38, 39]
    for causal, kv_len in ((True, None), (False, [30, 40]), (True, [7, 40])):
        _, dk, dv = _bwd(lib, q, k, v, do, 0.45, causal, kv_len)
        pk, pv = oracle.attention_bwd_kv_rows(q, k, v, do, 0.45, rows, causal=causal,
                                              kv_len=kv_len, nthreads=3, lib=lib)
        for part, full in ((pk, dk[:, :, rows]), (pv, dv[:, :, rows])):
            assert np.allclose(part, full, rtol=1e-12, atol=1e-13), (causal, kv_len)
        if kv_len is not None:        # keys at or past kv_len: no row sees them
            hidden = np.array(rows)[None, :] >= np.array(kv_len)[:, None]
            assert np.all(pk[hidden.nonzero()[0], :, hidden.nonzero()[1]] == 0.0)


PINS = [pin_bwd_finite_differences, pin_bwd_torch_autograd, pin_bwd_invariants,
        pin_bwd_zero_output_gradient, pin_bwd_bf16_inputs_equal_f64, pin_bwd_dq_rows_equal_full,
        pin_bwd_kv_rows_equal_full]


def failures(lib):
    out = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError as e:
            out.append(f"{pin.__name__}: {e}")
    return out

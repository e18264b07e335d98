"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

Each pin compares the oracle with something other than itself: a hand-derived
closed form, a limit of the softmax, an invariance of the definition, a
textbook library routine (torch's fp64 scaled_dot_product_attention), or the
independent blockwise online-softmax route. Each function takes the oracle
library handle (so the mutation test can run the same battery against planted
mistakes) and raises AssertionError on a mismatch.

Source of the facts: "FlashAttention (UR)", section "Problem of standard
attention" (the formula) and section "Online softmax" (running max and running
sum give the exact result); the softmax-row and limit properties are
mathematics of that formula.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle
from oracle.online import attention_online

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = 1e-12


def _num(x):
    if isinstance(x, str):
        table = {"ln2": math.log(2.0), "ln3": math.log(3.0), "ln4": math.log(4.0),
                 "-inf": -math.inf}
        return table[x]
    return float(x)


def _arr(rows):
    return np.array([[_num(x) for x in r] for r in rows], dtype=np.float64)


def _attn(lib, q, k, v, scale, causal=False, kv_len=None):
    return oracle.attention(q, k, v, scale, causal=causal, kv_len=kv_len, lib=lib)


def _rand(rng, B, H, N, d):
    return (rng.standard_normal((B, H, N, d)), rng.standard_normal((B, H, N, d)),
            rng.standard_normal((B, H, N, d)))


def _allowed(N, causal, kv_lim):
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    a = np.broadcast_to(j < kv_lim, (N, N))
    if causal:
        a = a & (j <= i)
    return a


# --------------------------------------------------------------------------
def pin_golden_closed_forms(lib):
    """Hand-derived worked examples (tests/golden/closed_form_cases.json)."""
    with open(os.path.join(GOLDEN, "closed_form_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q = _arr(c["q"])[None, None]
        k = _arr(c["k"])[None, None]
        v = _arr(c["v"])[None, None]
        scale = _num(c["scale"])
        variants = [("noncausal", False, None), ("causal", True, None),
                    ("kv_len_2", False, [2]), ("kv_len_0", False, [0])]
        for key, causal, kvl in variants:
            if key not in c:
                continue
            o, lse = _attn(lib, q, k, v, scale, causal, kvl)
            want_o = _arr(c[key]["o"])
            want_l = np.array([_num(x) for x in c[key]["lse"]])
            assert np.allclose(o[0, 0], want_o, atol=TOL, rtol=0), (c["name"], key, o[0, 0])
            assert np.array_equal(np.isinf(lse[0, 0]), np.isinf(want_l)), (c["name"], key)
            fin = np.isfinite(want_l)
            assert np.allclose(lse[0, 0][fin], want_l[fin], atol=TOL, rtol=0), (c["name"], key)


def pin_rows_sum_to_one(lib):
    """With V = identity (d = N), O equals the probability matrix P itself:
    every row must be non-negative, sum to 1, and be zero on hidden keys."""
    rng = np.random.default_rng(11)
    N = 24
    q = rng.standard_normal((2, 1, N, N))
    k = rng.standard_normal((2, 1, N, N))
    v = np.broadcast_to(np.eye(N), (2, 1, N, N)).copy()
    for causal, kvl in [(False, None), (True, None), (False, [N, 9]), (True, [5, 17])]:
        P, _ = _attn(lib, q, k, v, 0.3, causal, kvl)
        for b in range(2):
            lim = N if kvl is None else kvl[b]
            allowed = _allowed(N, causal, lim)
            assert np.all(P[b, 0] >= 0)
            assert np.allclose(P[b, 0].sum(axis=1), 1.0, atol=TOL, rtol=0)
            assert np.all(P[b, 0][~allowed] == 0.0)
            assert np.all(P[b, 0][allowed] > 0.0)


def pin_zero_query_means(lib):
    """Q = 0 makes every visible score 0: the softmax is uniform over the
    visible keys, so O_i is the mean of those V rows and lse_i = ln(count)."""
    rng = np.random.default_rng(12)
    B, H, N, d = 2, 2, 37, 5
    v = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, H, N, d))
    q = np.zeros((B, H, N, d))
    for causal, kvl in [(False, None), (True, None), (False, [20, 37]), (True, [11, 30])]:
        o, lse = _attn(lib, q, k, v, 0.7, causal, kvl)
        for b in range(B):
            lim = N if kvl is None else kvl[b]
            for i in range(N):
                hi = min(lim, i + 1) if causal else lim
                want = v[b, :, :hi].mean(axis=1)
                assert np.allclose(o[b, :, i], want, atol=TOL, rtol=0), (causal, kvl, b, i)
                assert np.allclose(lse[b, :, i], math.log(hi), atol=TOL, rtol=0)


def pin_dominant_key(lib):
    """A key aligned with a query and scaled up takes all the softmax weight
    for that query (limit of the softmax): O_i -> V_j*."""
    rng = np.random.default_rng(13)
    N, d = 16, 8
    q = rng.standard_normal((1, 1, N, d))
    k = rng.standard_normal((1, 1, N, d))
    v = rng.standard_normal((1, 1, N, d))
    pairs = [(3, 11), (9, 0), (15, 15)]          # (query row, dominant key)
    for axis, (i, j) in enumerate(pairs):        # orthogonal query directions
        q[0, 0, i] = 0.0
        q[0, 0, i, axis] = 2.0
        k[0, 0, j] = 0.0
        k[0, 0, j, axis] = 100.0                 # score 200 * scale ~ 70.7
    o, _ = _attn(lib, q, k, v, 1.0 / math.sqrt(d))
    for i, j in pairs:
        assert np.allclose(o[0, 0, i], v[0, 0, j], atol=1e-9, rtol=0), (i, j)


def pin_causal_row_zero(lib):
    """Causal row 0 sees only key 0: O_0 = V_0 and lse_0 = scale * <q_0, k_0>."""
    rng = np.random.default_rng(14)
    B, H, N, d = 2, 3, 19, 7
    q, k, v = _rand(rng, B, H, N, d)
    o, lse = _attn(lib, q, k, v, 0.4, causal=True)
    assert np.allclose(o[:, :, 0], v[:, :, 0], atol=TOL, rtol=0)
    want = 0.4 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0])
    assert np.allclose(lse[:, :, 0], want, atol=TOL, rtol=0)


def pin_constant_values(lib):
    """V constant along keys makes O that constant (the weights sum to 1)."""
    rng = np.random.default_rng(15)
    B, H, N, d = 1, 2, 33, 4
    q, k, _ = _rand(rng, B, H, N, d)
    c = np.array([1.5, -2.0, 0.25, 7.0])
    v = np.broadcast_to(c, (B, H, N, d)).copy()
    for causal, kvl in [(False, None), (True, None), (False, [10])]:
        o, _ = _attn(lib, q, k, v, 0.5, causal, kvl)
        assert np.allclose(o, np.broadcast_to(c, o.shape), atol=TOL, rtol=0)


def pin_key_permutation(lib):
    """Without a causal mask, permuting keys and values together leaves O and
    lse unchanged; permuting queries permutes the output rows."""
    rng = np.random.default_rng(16)
    B, H, N, d = 1, 2, 29, 6
    q, k, v = _rand(rng, B, H, N, d)
    perm = rng.permutation(N)
    o1, l1 = _attn(lib, q, k, v, 0.35)
    o2, l2 = _attn(lib, q, k[:, :, perm], v[:, :, perm], 0.35)
    assert np.allclose(o1, o2, atol=TOL, rtol=0)
    assert np.allclose(l1, l2, atol=TOL, rtol=0)
    o3, l3 = _attn(lib, q[:, :, perm], k, v, 0.35)
    assert np.allclose(o3, o1[:, :, perm], atol=TOL, rtol=0)
    assert np.allclose(l3, l1[:, :, perm], atol=TOL, rtol=0)


def pin_torch_sdpa(lib):
    """Special case that reduces to a library routine: torch's CPU fp64
    scaled_dot_product_attention with a boolean mask (True = visible)."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(17)
    B, H, N, d = 2, 3, 45, 16
    q, k, v = _rand(rng, B, H, N, d)
    for causal, kvl in [(False, None), (True, None), (False, [30, 45]), (True, [7, 40])]:
        o, _ = _attn(lib, q, k, v, 0.2, causal, kvl)
        mask = np.zeros((B, 1, N, N), dtype=bool)
        for b in range(B):
            mask[b, 0] = _allowed(N, causal, N if kvl is None else kvl[b])
        ref = F.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
            attn_mask=torch.from_numpy(mask), scale=0.2).numpy()
        assert np.allclose(o, ref, atol=1e-12, rtol=0), (causal, kvl)


def pin_online_equals_full(lib):
    """The blockwise online softmax (running max and sum, rescaled per block)
    gives the same result as the two-pass full softmax."""
    rng = np.random.default_rng(18)
    for N in (1, 2, 7, 64, 100, 300):
        q, k, v = _rand(rng, 1, 2, N, 8)
        q = q * 3.0  # peaky rows exercise the rescaling
        for causal, kvl in [(False, None), (True, None), (False, [max(1, N // 3)])]:
            o, lse = _attn(lib, q, k, v, 0.5, causal, kvl)
            for blk in (1, 7, 16, 64):
                o2, l2 = attention_online(q, k, v, 0.5, causal, kvl, block=blk)
                assert np.allclose(o, o2, atol=TOL, rtol=0), (N, causal, kvl, blk)
                assert np.allclose(lse, l2, atol=TOL, rtol=0), (N, causal, kvl, blk)


def pin_no_visible_key(lib):
    """kv_len = 0: every row has no visible key -> O = 0, lse = -inf."""
    rng = np.random.default_rng(19)
    q, k, v = _rand(rng, 2, 1, 9, 4)
    o, lse = _attn(lib, q, k, v, 1.0, False, [0, 9])
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


def pin_grouped_heads_equal_repeated_heads(lib):
    """Grouped/multi-query attention is multi-head attention whose K/V heads are
    repeated for each group of query heads (query head h uses K/V head
    h // (H // Hkv)); with Hkv == H nothing changes."""
    rng = np.random.default_rng(20)
    B, H, N, d = 2, 6, 23, 8
    q = rng.standard_normal((B, H, N, d))
    for Hkv in (1, 2, 3, 6):
        k = rng.standard_normal((B, Hkv, N, d))
        v = rng.standard_normal((B, Hkv, N, d))
        g = H // Hkv
        k_rep = np.repeat(k, g, axis=1)
        v_rep = np.repeat(v, g, axis=1)
        for causal, kvl in [(False, None), (True, [23, 9])]:
            o, lse = _attn(lib, q, k, v, 0.3, causal, kvl)
            o2, l2 = _attn(lib, q, k_rep, v_rep, 0.3, causal, kvl)
            assert np.array_equal(o, o2) and np.array_equal(lse, l2), (Hkv, causal)
            if Hkv == 1:   # every query head sees the same keys: permuting heads commutes
                perm = rng.permutation(H)
                o3, _ = _attn(lib, q[:, perm], k, v, 0.3, causal, kvl)
                assert np.allclose(o3, o[:, perm], atol=TOL, rtol=0)


def pin_fewer_queries_are_the_last_rows(lib):
    """With Nq < Nk queries (query row i standing at key position i + Nk - Nq),
    each output row equals the matching row of full self-attention over the
    Nk positions whose last Nq queries are these (the mask and the keys seen
    are the same)."""
    rng = np.random.default_rng(21)
    B, H, Nk, d = 2, 3, 41, 8
    q_full = rng.standard_normal((B, H, Nk, d))
    k = rng.standard_normal((B, 1, Nk, d))
    v = rng.standard_normal((B, 1, Nk, d))
    for Nq in (1, 5, 41):
        for causal, kvl in [(True, None), (False, None), (True, [41, 30]), (False, [12, 41])]:
            o_full, l_full = _attn(lib, q_full, k, v, 0.45, causal, kvl)
            o, lse = _attn(lib, q_full[:, :, Nk - Nq:], k, v, 0.45, causal, kvl)
            assert np.array_equal(o, o_full[:, :, Nk - Nq:]), (Nq, causal, kvl)
            assert np.array_equal(lse, l_full[:, :, Nk - Nq:]), (Nq, causal, kvl)
    # a single causal query at the last position sees every key: the non-causal answer
    o1, _ = _attn(lib, q_full[:, :, -1:], k, v, 0.45, True)
    o2, _ = _attn(lib, q_full[:, :, -1:], k, v, 0.45, False)
    assert np.array_equal(o1, o2)


ALL_PINS = [
    pin_golden_closed_forms,
    pin_rows_sum_to_one,
    pin_zero_query_means,
    pin_dominant_key,
    pin_causal_row_zero,
    pin_constant_values,
    pin_key_permutation,
    pin_torch_sdpa,
    pin_online_equals_full,
    pin_no_visible_key,
    pin_grouped_heads_equal_repeated_heads,
    pin_fewer_queries_are_the_last_rows,
]


def failures(lib):
    """Run every pin; return the names of those that fail (or crash)."""
    bad = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except Exception:  # noqa: BLE001 - any failure counts
            bad.append(pin.__name__)
    return bad

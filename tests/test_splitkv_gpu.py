"""GPU parity of the split-KV forward (fa_fwd_splitkv) against the fp64 oracle.

Few query rows against many keys: q [B,H,Nq,d], k, v [B,H_kv,Nk,d] with
Nq <= Nk, query row i at key position i + Nk - Nq. The keys of every row are
cut into num_splits ranges whose partial results are merged by log-sum-exp,
and the query heads sharing a K/V head are packed into one tile. Tolerances
are those of the square forward (tests/test_parity_gpu.py).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.test_parity_gpu import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_18_b200 as fa
    from io_aware_exact_18_b200 import build
    build.build()
    fa.load_library()
    return fa


def run_splitkv(fa, q, k, v, causal, splits, kv_len=None, poison_ws=True):
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    kvd = None if kv_len is None else kv_len.to(dev)
    B, H, Nq, d = q.shape
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=dev)
    ws = None
    if splits is not None:
        need = fa.fa_splitkv_workspace_bytes(B, H, Nq, d, splits)
        if need:
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
            if poison_ws:   # the workspace needs no initialisation
                ws.view(torch.float32)[: need // 4].fill_(float("nan"))
    fa.decode_attention(qd, kd, vd, causal=causal, kv_len=kvd, num_splits=splits, out=out,
                        lse=lse, workspace=ws)
    st = fa.fa_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return out, lse


def check(fa, q, k, v, causal, splits, kv_len=None, what=""):
    out, lse = run_splitkv(fa, q, k, v, causal, splits, kv_len)
    d = q.shape[-1]
    o_ref, lse_ref = oracle.attention(q, k, v, 1.0 / math.sqrt(d), causal=causal, kv_len=kv_len)
    return compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref,
                   what)


@pytest.mark.parametrize("splits", [1, 2, 7, None])
@pytest.mark.parametrize("Nk", [1, 127, 128, 1000, 4099])
def test_decode_one_query(fa, Nk, splits):
    """One query row per (b, h) against Nk keys; grouped heads packed 4 per tile."""
    q, k, v, _ = workloads.make_qkv(3, 8, 2, 1, Nk, 128, seed=2000 + Nk)
    for causal in (False, True):
        check(fa, q, k, v, causal, splits, what=f"Nk={Nk} splits={splits} causal={causal}")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("H,H_kv", [(8, 2), (6, 1), (4, 4), (12, 4)])
@pytest.mark.parametrize("Nq", [7, 128, 130])
def test_short_queries_all_head_layouts(fa, Nq, H, H_kv, d):
    """Several query rows (a ragged row block when 128 / group does not divide
    Nq), causal offset Nk - Nq, every head-group size, every head dim."""
    Nk = 1000
    q, k, v, _ = workloads.make_qkv(2, H, H_kv, Nq, Nk, d, seed=3000 + Nq + H + H_kv + d)
    for causal in (False, True):
        for splits in (1, 3):
            check(fa, q, k, v, causal, splits,
                  what=f"Nq={Nq} H={H} H_kv={H_kv} d={d} causal={causal} splits={splits}")


def test_key_padding_with_empty_ranges(fa):
    """Per-sequence cache lengths, including 0 (every key hidden: O = 0 and
    lse = -inf) and lengths shorter than the number of ranges (empty ranges)."""
    B, H, H_kv, Nq, Nk, d = 5, 8, 2, 3, 2048, 128
    q, k, v, _ = workloads.make_qkv(B, H, H_kv, Nq, Nk, d, seed=4242)
    kv_len = torch.tensor([0, 1, 130, 1500, 2048], dtype=torch.int32)
    for causal in (False, True):
        for splits in (1, 4, 16, 33):
            check(fa, q, k, v, causal, splits, kv_len,
                  what=f"kv_len causal={causal} splits={splits}")


def test_prefill_chunk_against_cache(fa):
    """A 300-row chunk of new queries against a 2300-key cache (causal offset
    2000), grouped heads packed 4 per tile (32 rows per head per tile)."""
    q, k, v, _ = workloads.make_qkv(1, 8, 2, 300, 2300, 128, seed=77)
    for splits in (1, 5):
        check(fa, q, k, v, True, splits, what=f"chunk splits={splits}")


def test_square_single_range_matches_fa_fwd_bitwise(fa):
    """Nq == Nk, one range, H_kv == H: the same tiles as fa_fwd, so the same bits."""
    q, k, v, _ = workloads.make_qkv(2, 4, 4, 777, 777, 128, seed=5)
    dev = torch.device("cuda:0")
    for causal in (False, True):
        o1, l1 = run_splitkv(fa, q, k, v, causal, 1)
        o2, l2 = fa.attention(q.to(dev), k.to(dev), v.to(dev), causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_workload_full_size(fa):
    """The decode workload the benchmark times, every row checked, at the
    split count the benchmark uses (the library's default) and at 8 ranges."""
    w = workloads.DECODE_WORKLOADS[0]
    q, k, v, _ = workloads.make_qkv(w.B, w.H, w.H_kv, w.Nq, w.Nk, w.d, seed=w.seed)
    splits = fa.fa_splitkv_default_splits(w.B, w.H, w.H_kv, w.Nq, w.Nk, w.d)
    for sp in sorted({splits, 8}):
        check(fa, q, k, v, w.causal, sp, what=f"{w.name} splits={sp}")


def test_long_cache_decode_workload_sampled(fa):
    """The 128K-key decode workload at the default (split) range count, all
    32 heads' single rows checked against the oracle."""
    w = workloads.DECODE_WORKLOADS[1]
    q, k, v, _ = workloads.make_qkv(w.B, w.H, w.H_kv, w.Nq, w.Nk, w.d, seed=w.seed)
    splits = fa.fa_splitkv_default_splits(w.B, w.H, w.H_kv, w.Nq, w.Nk, w.d)
    assert splits > 1
    check(fa, q, k, v, w.causal, splits, what=f"{w.name} splits={splits}")


def test_default_splits_fill_the_device(fa):
    """One long-context head group needs many ranges; a large batch needs one."""
    assert fa.fa_splitkv_default_splits(1, 32, 8, 1, 131072, 128) >= 8
    assert fa.fa_splitkv_default_splits(64, 32, 8, 1, 8192, 128) == 1


def test_splits_are_deterministic(fa):
    q, k, v, _ = workloads.make_qkv(2, 8, 2, 5, 3000, 128, seed=9)
    a = run_splitkv(fa, q, k, v, True, 6)
    b = run_splitkv(fa, q, k, v, True, 6, poison_ws=False)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_splitkv_guard_regions_untouched(fa):
    """Writes stay inside O and lse: sentinels around both survive."""
    B, H, H_kv, Nq, Nk, d = 2, 8, 2, 3, 1000, 128
    q, k, v, _ = workloads.make_qkv(B, H, H_kv, Nq, Nk, d, seed=10)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    n_o, n_l, pad = B * H * Nq * d, B * H * Nq, 4096
    o_buf = torch.full((n_o + 2 * pad,), 7.0, dtype=torch.bfloat16, device=dev)
    l_buf = torch.full((n_l + 2 * pad,), 7.0, dtype=torch.float32, device=dev)
    out = o_buf[pad:pad + n_o].view(B, H, Nq, d)
    lse = l_buf[pad:pad + n_l].view(B, H, Nq)
    fa.decode_attention(qd, kd, vd, causal=True, num_splits=4, out=out, lse=lse)
    torch.cuda.synchronize()
    for buf, n in ((o_buf, n_o), (l_buf, n_l)):
        assert torch.all(buf[:pad] == 7.0) and torch.all(buf[pad + n:] == 7.0)


def test_decode_million_key_cache(fa):
    """One query row per head against 2^20 keys (8192 key tiles), at the
    library's default range count: every row against the oracle."""
    B, H, H_kv, Nq, Nk, d = 1, 16, 4, 1, 1 << 20, 128
    q, k, v, _ = workloads.make_qkv(B, H, H_kv, Nq, Nk, d, seed=20)
    splits = fa.fa_splitkv_default_splits(B, H, H_kv, Nq, Nk, d)
    assert splits > 1
    check(fa, q, k, v, True, splits, what=f"Nk=2^20 splits={splits}")

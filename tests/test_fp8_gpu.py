"""GPU parity of the e4m3 forward (fa_fwd_fp8 at d = 64, 128 and 256, and the
split-KV form fa_fwd_splitkv_fp8) against the fp64 oracle on the dequantized
inputs (oracle.fp8.attention_fp8).

Tolerance, derived from the arithmetic: scores are exact (products of e4m3
values are exact in fp32; accumulation is fp32), so lse keeps the bf16 path's
bound |d lse| / max(|lse_ref|, 1) <= 1e-3. Each probability is rounded to
e4m3 before the P.V product: relative error at most 2^-4 (3 mantissa bits).
With weights summing to one after normalisation, |dO| <= 2^-4 * max|V|, plus
bf16 rounding of O (2^-8 * max|O|): that is the element-wise bound. The mean
error, an average of independent roundings, is bounded by 2^-7 * max|V|.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import fp8 as ofp8

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


def run_fp8(fa, q8, k8, v8, sc, causal, kv_len=None, cache=False, splits=None, scale=None):
    """One e4m3 launch: square (fa_fwd_fp8) or, with cache=True, through the
    split-KV entry (Nq <= Nk, query heads of a K/V group packed)."""
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev) for x in (q8, k8, v8))
    kvd = None if kv_len is None else kv_len.to(dev)
    B, H, N, d = q8.shape
    out = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    if cache:
        fa.decode_attention_fp8(qd, kd, vd, *sc, scale=scale, causal=causal, kv_len=kvd,
                                num_splits=splits, out=out, lse=lse)
    else:
        fa.attention_fp8(qd, kd, vd, *sc, scale=scale, causal=causal, kv_len=kvd, out=out,
                         lse=lse)
    st = fa.fa_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def compare_fp8(o, lse, o_ref, lse_ref, vmax, what, rows=None):
    if rows is not None:
        o, lse = o[:, :, rows], lse[:, :, rows]
    assert not np.isnan(o).any() and not np.isnan(lse).any(), f"{what}: unwritten output"
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), dead), f"{what}: -inf pattern differs"
    err = np.abs(o - o_ref)
    bound = 2.0 ** -4 * vmax + 2.0 ** -8 * np.abs(o_ref).max()
    assert err.max() <= bound, f"{what}: max|dO| {err.max():.3e} > {bound:.3e}"
    assert err.mean() <= 2.0 ** -7 * vmax, f"{what}: mean|dO| {err.mean():.3e}"
    live = ~dead
    rel = np.abs(lse[live] - lse_ref[live]) / np.maximum(np.abs(lse_ref[live]), 1.0)
    assert rel.size == 0 or rel.max() <= 1e-3, f"{what}: lse rel err {rel.max():.3e}"
    return float(err.max() / vmax), float(err.mean() / vmax)


def check_fp8(fa, B, H, H_kv, N, causal, seed, kv_len_range=None, rows=None, d=128,
              Nk=None, splits=None):
    """Parity of one e4m3 configuration. Nk given: the split-KV entry with N
    query rows against Nk keys (splits key ranges, None for the library's
    choice); else the square entry."""
    cache = Nk is not None
    q8, k8, v8, sc, kvl = workloads.make_fp8_inputs(B, H, H_kv, N, d, seed, kv_len_range,
                                                    Nk=Nk)
    o, lse = run_fp8(fa, q8, k8, v8, sc, causal, kvl, cache=cache, splits=splits)
    o_ref, lse_ref = ofp8.attention_fp8(q8, k8, v8, *sc, 1.0 / math.sqrt(d), causal=causal,
                                        kv_len=kvl, rows=rows)
    vmax = float(np.abs(ofp8.decode_e4m3(v8.view(torch.uint8).numpy())).max() * sc[2])
    what = f"B{B} H{H}/{H_kv} N{N} Nk{Nk} d{d} c{causal} splits={splits}"
    return compare_fp8(o, lse, o_ref, lse_ref, vmax, what, rows)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 128, 300, 1024])
def test_fp8_lengths(fa, N, causal):
    check_fp8(fa, 2, 2, 2, N, causal, seed=6000 + N + causal)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_grouped_heads_and_padding(fa, causal):
    check_fp8(fa, 2, 8, 2, 700, causal, seed=6100 + causal, kv_len_range=(0, 700))


def test_fp8_full_size_sampled(fa):
    """The long-context shape (B1 H32 N16384 causal) in one launch, checked on
    sampled rows of every head."""
    N = 16384
    rows = workloads.sample_rows(N, seed=61, n_random=48, edge=16)
    check_fp8(fa, 1, 32, 32, N, True, seed=6200, rows=rows)


def test_fp8_is_deterministic(fa):
    q8, k8, v8, sc, _ = workloads.make_fp8_inputs(1, 4, 4, 999, 128, 6300)
    a = run_fp8(fa, q8, k8, v8, sc, True)
    b = run_fp8(fa, q8, k8, v8, sc, True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 129, 300, 1024])
def test_fp8_head_dim_256(fa, N, causal):
    """d = 256: one query tile per unit, two 128-byte column blocks per row."""
    check_fp8(fa, 2, 2, 2, N, causal, seed=6400 + N + causal, d=256)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_head_dim_256_grouped_heads_and_padding(fa, causal):
    check_fp8(fa, 2, 4, 2, 600, causal, seed=6500 + causal, kv_len_range=(0, 600), d=256)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("Nq,Nk,H,H_kv,splits,causal", [
    (1, 4096, 8, 2, None, False),       # one-token decoding, the library's key ranges
    (1, 1000, 4, 4, 3, True),           # ragged key count, three ranges
    (16, 777, 8, 1, 2, True),           # multi-query: 8 heads packed, 16 rows each
    (200, 200, 4, 2, 1, True),          # Nq == Nk through the general kernel
    (130, 2048, 2, 1, 5, False),        # two row blocks per head pair
])
def test_fp8_splitkv(fa, d, Nq, Nk, H, H_kv, splits, causal):
    """The e4m3 split-KV entry: Nq <= Nk with the causal offset Nk - Nq,
    grouped heads packed into one tile, key ranges merged by their lse."""
    check_fp8(fa, 2, H, H_kv, Nq, causal, seed=6600 + Nq + d, d=d, Nk=Nk, splits=splits)


@pytest.mark.parametrize("d", [128, 256])
def test_fp8_splitkv_key_padding(fa, d):
    """kv_len per batch (0 included: empty rows give lse = -inf and O = 0)."""
    q8, k8, v8, sc, _ = workloads.make_fp8_inputs(3, 4, 2, 5, d, 6700 + d, Nk=900)
    kvl = torch.tensor([0, 1, 637], dtype=torch.int32)
    o, lse = run_fp8(fa, q8, k8, v8, sc, False, kvl, cache=True, splits=4)
    o_ref, lse_ref = ofp8.attention_fp8(q8, k8, v8, *sc, 1.0 / math.sqrt(d), kv_len=kvl)
    vmax = float(np.abs(ofp8.decode_e4m3(v8.view(torch.uint8).numpy())).max() * sc[2])
    compare_fp8(o, lse, o_ref, lse_ref, vmax, f"kv_len padding d{d}")
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse[0]))



@pytest.mark.parametrize("H,H_kv,Nq,causal", [
    (8, 2, 1, True),      # 4 heads per K/V head: the transposed decoding tile
    (8, 1, 1, False),     # 8 columns, the tile's limit
    (4, 4, 2, True),      # one head per group, 2 rows
    (2, 1, 4, False),     # 8 columns from 2 heads x 4 rows
    (1, 1, 9, True),      # 9 columns: the general kernel
])
def test_fp8_decoding_tile(fa, H, H_kv, Nq, causal):
    """e4m3 decoding through fa_fwd_splitkv_fp8 at d = 128, on both sides of the
    transposed tile's 8-column limit, at the default and two fixed range counts."""
    for splits in (None, 1, 3):
        check_fp8(fa, 2, H, H_kv, Nq, causal, seed=6800 + 7 * H + Nq, d=128, Nk=3000,
                  splits=splits)


def test_fp8_decoding_reference_moves_every_tile(fa):
    """e4m3 scores that grow by more than 8 log2 units from one key tile to the
    next (q = 32 and every key of tile t equal to 2t along one axis, exact in
    e4m3), so every column's reference maximum moves at every tile."""
    B, H, H_kv, Nq, Nk, d = 1, 4, 1, 1, 11 * 128, 128
    q = torch.zeros(B, H, Nq, d)
    q[..., 0] = 32.0
    k = torch.zeros(B, H_kv, Nk, d)
    k[..., 0] = 2.0 * (torch.arange(Nk) // 128).float()
    g = torch.Generator().manual_seed(4)
    v = torch.randn(B, H_kv, Nk, d, generator=g)
    q8, k8, v8 = (x.to(torch.float8_e4m3fn) for x in (q, k, v))
    assert 32 * 2 / math.sqrt(d) * math.log2(math.e) > 8
    sc = (1.0, 1.0, 1.0)
    for splits in (1, 3):
        o, lse = run_fp8(fa, q8, k8, v8, sc, False, cache=True, splits=splits)
        o_ref, lse_ref = ofp8.attention_fp8(q8, k8, v8, *sc, 1.0 / math.sqrt(d))
        vmax = float(np.abs(ofp8.decode_e4m3(v8.view(torch.uint8).numpy())).max())
        compare_fp8(o, lse, o_ref, lse_ref, vmax, f"e4m3 moving reference splits={splits}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 129, 300, 1024])
def test_fp8_head_dim_64(fa, N, causal):
    """d = 64: a row is 64 bytes, stored with the 64-byte swizzle (TMA box and
    tcgen05 descriptors), two query tiles per unit."""
    check_fp8(fa, 2, 2, 2, N, causal, seed=6900 + N + causal, d=64)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_head_dim_64_grouped_heads_padding_and_cache(fa, causal):
    check_fp8(fa, 2, 8, 2, 700, causal, seed=6950 + causal, kv_len_range=(0, 700), d=64)
    for splits in (None, 1, 3):
        check_fp8(fa, 2, 8, 2, 5, causal, seed=6960 + causal, d=64, Nk=2000, splits=splits)
        check_fp8(fa, 1, 4, 4, 200, causal, seed=6970 + causal, d=64, Nk=1000, splits=splits)



@pytest.mark.parametrize("d", [64, 128, 256])
def test_fp8_reference_moves_square(fa, d):
    """e4m3 scores that climb tile by tile at different rates within a warp.
    Query row i carries a_i in {0, 1/8, 1/2, 1} (cycling) in column 0, key j
    carries 48 * (j // 128) there (exact in e4m3 up to 288), the other columns
    small values; with scale 1/8 a key tile raises a row's scores by 8.66 a_i
    log2 units, so rows with a_i = 1 move their reference maximum (threshold 8)
    on every later tile, a_i = 1/2 every other tile, the rest never. Without
    the moves, tile 6's probabilities for a_i = 1 would be 2^52 and saturate at
    448, so O within the e4m3 bound shows the rescale of O and l ran."""
    N, scale = 7 * 128, 0.125
    g = torch.Generator().manual_seed(5)
    q = 0.25 * torch.randn(1, 2, N, d, generator=g)
    k = 0.25 * torch.randn(1, 2, N, d, generator=g)
    v = torch.randn(1, 2, N, d, generator=g)
    q[..., 0] = torch.tensor([0.0, 0.125, 0.5, 1.0]).repeat(N // 4)
    k[..., 0] = 48.0 * (torch.arange(N) // 128).float()
    q8, k8, v8 = (x.to(torch.float8_e4m3fn) for x in (q, k, v))
    assert torch.equal(k8[0, 0, :, 0].float(), 48.0 * (torch.arange(N) // 128).float())
    assert 48 * scale * math.log2(math.e) > 8
    sc = (1.0, 1.0, 1.0)
    vmax = float(np.abs(ofp8.decode_e4m3(v8.view(torch.uint8).numpy())).max())
    for causal in (False, True):
        o, lse = run_fp8(fa, q8, k8, v8, sc, causal, scale=scale)
        o_ref, lse_ref = ofp8.attention_fp8(q8, k8, v8, *sc, scale, causal=causal)
        compare_fp8(o, lse, o_ref, lse_ref, vmax, f"e4m3 climbing scores d={d} causal={causal}")

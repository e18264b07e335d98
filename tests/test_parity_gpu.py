"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances (bf16 inputs, fp32 accumulation, bf16 output), per element of O
against the oracle: max |dO| <= 2e-2 and mean |dO| <= 2e-3; for the
log-sum-exp, |d lse| / max(|lse_ref|, 1) <= 1e-3 (the relative form is
ill-posed where lse is near 0, e.g. causal row 0, hence the floor of 1).
Rows with no visible key must give O = 0 and lse = -inf exactly.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_REL = 1e-3


def _fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_18_b200 as fa
    from io_aware_exact_18_b200 import build
    build.build()
    fa.load_library()
    return fa


@pytest.fixture(scope="module")
def fa():
    return _fa()


def run_gpu(fa, q, k, v, causal, kv_len=None, scale=None):
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    kvd = None if kv_len is None else kv_len.to(dev)
    B, H, N, d = q.shape
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    fa.attention(qd, kd, vd, scale=scale, causal=causal, kv_len=kvd, out=out, lse=lse)
    st = fa.fa_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def compare(o, lse, o_ref, lse_ref, what=""):
    assert not np.isnan(o).any(), f"{what}: unwritten (NaN) output elements"
    assert not np.isnan(lse).any(), f"{what}: unwritten (NaN) lse elements"
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), dead), f"{what}: -inf pattern differs"
    if dead.any():
        assert np.all(o[dead] == 0.0), f"{what}: rows with no visible key must be 0"
    err = np.abs(o - o_ref)
    assert err.max() <= MAX_ABS, f"{what}: max|dO| = {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean|dO| = {err.mean():.3e}"
    live = ~dead
    if live.any():
        rel = np.abs(lse[live] - lse_ref[live]) / np.maximum(np.abs(lse_ref[live]), 1.0)
        assert rel.max() <= LSE_REL, f"{what}: lse rel err {rel.max():.3e}"
    return float(err.max()), float(err.mean())


def check_full(fa, q, k, v, causal, kv_len=None, scale=None, what=""):
    d = q.shape[-1]
    sc = (1.0 / math.sqrt(d)) if scale is None else scale
    o, lse = run_gpu(fa, q, k, v, causal, kv_len, scale=sc)
    o_ref, lse_ref = oracle.attention(q, k, v, sc, causal=causal, kv_len=kv_len)
    return compare(o, lse, o_ref, lse_ref, what)


# ----------------------------------------------------------------- workloads
@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_workload_full(fa, idx):
    """Every element of every workload against the oracle, each at its full
    size in the launch the benchmark times: the tiny case, BERT-large-shaped
    key padding, GPT-2-shaped causal, the long-range case whose queries are
    scaled by 4 (peaky rows that stress the running maximum and rescaling of
    the online softmax) and the long-context case (about 2.2 TFLOP of fp64
    oracle work, some 40 s on 16 host cores)."""
    w = workloads.get(idx)
    q, k, v, kv_len = workloads.make_inputs(w)
    check_full(fa, q, k, v, w.causal, kv_len, w.scale, w.name)


# ----------------------------------------------------------------- ragged / edge shapes
RAGGED = [1, 17, 127, 128, 129, 255, 256, 257, 300, 383, 513]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", RAGGED)
def test_ragged_lengths(fa, N, causal, d):
    q, k, v, _ = workloads.make_custom(2, 2, N, d, seed=1000 + N + d + 7 * causal)
    check_full(fa, q, k, v, causal, what=f"N={N} causal={causal} d={d}")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_key_padding_edges(fa, causal, d):
    N = 300
    q, k, v, _ = workloads.make_custom(6, 2, N, d, seed=77 + d)
    kv_len = torch.tensor([0, 1, 127, 128, 299, 5000], dtype=torch.int32)  # 5000 clamps to N
    check_full(fa, q, k, v, causal, kv_len, what=f"kv_len edges causal={causal} d={d}")


@pytest.mark.parametrize("causal", [False, True])
def test_persistent_mixed_units(fa, causal):
    """Far more work units than SMs, so CTAs take over units of CTAs that have
    not started; the units mix idle query tiles (N = 300 leaves the second
    tile of the last pair empty), sequences whose keys are all hidden
    (kv_len = 0) and short ones, so every per-unit hand-off is exercised."""
    B, H, N, d = 40, 8, 300, 64
    q, k, v, _ = workloads.make_custom(B, H, N, d, seed=321 + causal)
    g = torch.Generator().manual_seed(5)
    kv_len = torch.randint(0, N + 1, (B,), generator=g).to(torch.int32)
    kv_len[::7] = 0
    kv_len[1::7] = 1
    check_full(fa, q, k, v, causal, kv_len, what=f"persistent mixed causal={causal}")


def test_persistent_many_heads_d128(fa):
    q, k, v, _ = workloads.make_custom(3, 100, 520, 128, seed=99)
    check_full(fa, q, k, v, True, what="persistent 300 heads d=128")


@pytest.mark.parametrize("causal", [False, True])
def test_head_dim_256_long(fa, causal):
    """d = 256 (one query tile per unit, double-buffered scores) over many key
    tiles and units, with mixed key-padding lengths."""
    B, H, N, d = 4, 12, 1100, 256
    q, k, v, _ = workloads.make_custom(B, H, N, d, seed=256 + causal)
    kv_len = torch.tensor([1100, 700, 1, 0], dtype=torch.int32)
    check_full(fa, q, k, v, causal, kv_len, what=f"d=256 causal={causal}")


def test_head_dim_256_sampled_full_size(fa):
    """Long sequence at d = 256: sampled rows against the oracle."""
    B, H, N, d = 1, 4, 8192, 256
    q, k, v, _ = workloads.make_custom(B, H, N, d, seed=2560)
    o, lse = run_gpu(fa, q, k, v, True)
    rows = workloads.sample_rows(N, seed=7, n_random=48, edge=48)
    o_ref, lse_ref = oracle.attention(q, k, v, 1 / math.sqrt(d), causal=True, rows=rows)
    compare(o[:, :, rows], lse[:, :, rows], o_ref, lse_ref, "d=256 N=8192 causal")


@pytest.mark.parametrize("H,H_kv", [(8, 2), (6, 1), (4, 4)])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_grouped_and_multi_query(fa, H, H_kv, d, causal):
    """K/V heads shared by groups of query heads (H_kv = 1: multi-query)."""
    B, N = 3, 333
    q, k, v, _ = workloads.make_qkv(B, H, H_kv, N, N, d, seed=1000 + H * 10 + H_kv + d + causal)
    kv_len = torch.tensor([333, 200, 0], dtype=torch.int32)
    check_full(fa, q, k, v, causal, kv_len, what=f"H={H} H_kv={H_kv} d={d} causal={causal}")
    check_full(fa, q, k, v, causal, None, what=f"H={H} H_kv={H_kv} d={d} causal={causal}")


def test_grouped_heads_sampled_full_size(fa):
    """The grouped-heads long-context launch the benchmark measures (B1 H32
    H_kv8 N16384 d128 causal): sampled rows of every head against the oracle."""
    B, H, H_kv, N, d = 1, 32, 8, 16384, 128
    q, k, v, _ = workloads.make_qkv(B, H, H_kv, N, N, d, seed=3208)
    o, lse = run_gpu(fa, q, k, v, True)
    rows = workloads.sample_rows(N, seed=8, n_random=32, edge=16)
    o_ref, lse_ref = oracle.attention(q, k, v, 1 / math.sqrt(d), causal=True, rows=rows)
    compare(o[:, :, rows], lse[:, :, rows], o_ref, lse_ref, "H32 H_kv8 N16384 causal")


def test_peaky_rows_rescale(fa):
    """Large |scores| (Q x 8, far from unit-normal scores): rows are dominated by
    one or two keys, whose weights the running reference maximum of the kernel
    does not bring to exactly 1, so their bf16 rounding (up to 2^-8 relative)
    would reach O if O were divided by the exact sum of the probabilities. The
    kernel divides O by the sum of the probabilities as rounded for the P.V
    product instead, which keeps such a row at its dominant V row to within the
    output rounding, and the benchmark spec's bound holds: max |dO| <= 2e-2,
    mean |dO| <= 2e-3, lse within 1e-3 (measured on a B200: 1.25e-2; 2.28e-2
    with the exact sum as the divisor; 1.66e-2 for a kernel with an exact running
    maximum)."""
    q, k, v, _ = workloads.make_custom(1, 4, 1024, 128, seed=9, q_mult=8.0)
    for causal in (False, True):
        o, lse = run_gpu(fa, q, k, v, causal, scale=1 / math.sqrt(128))
        o_ref, lse_ref = oracle.attention(q, k, v, 1 / math.sqrt(128), causal=causal)
        err = compare(o, lse, o_ref, lse_ref, f"Qx8 causal={causal}")
        print(f"Qx8 causal={causal}: max|dO| {err[0]:.4e} mean|dO| {err[1]:.4e}")


LOG2E = 1.4426950408889634


def reference_moves(q, k, scale, causal, tile=128):
    """Per query row, how many key tiles move the reference maximum of the
    two-query-tile kernel (d <= 128): the row's first key tile sets the
    reference m to its maximum; a later tile whose maximum exceeds m by more
    than 64 in log2 units (some probability exp2((s - m) * scale * log2 e)
    would pass 2^64) makes the row take that maximum, rescaling O and l before
    the tile is exponentiated. Evaluated in fp64 from the bf16 inputs of one
    head."""
    s = (q[0, 0].double() @ k[0, 0].double().T).numpy() * scale * LOG2E
    n = s.shape[0]
    counts = np.zeros(n, dtype=int)
    for i in range(n):
        row = s[i, :(i + 1 if causal else n)]
        m = row[:tile].max()
        for t0 in range(tile, row.shape[0], tile):
            part = row[t0:t0 + tile]
            if part.max() - m > 64.0:
                m = part.max()
                counts[i] += 1
    return counts


def reference_redos(q, k, scale, causal, tile=128):
    """The same count for the one-query-tile kernel (d = 256): the first key
    tile sets m to its maximum; a later tile is exponentiated against m and,
    if its probabilities exp2((s - m) * scale * log2 e) sum past 2^64, the row
    takes the larger of m and the tile's maximum, rescales O and l, and redoes
    the tile."""
    s = (q[0, 0].double() @ k[0, 0].double().T).numpy() * scale * LOG2E
    n = s.shape[0]
    counts = np.zeros(n, dtype=int)
    for i in range(n):
        row = s[i, :(i + 1 if causal else n)]
        m = row[:tile].max()
        for t0 in range(tile, row.shape[0], tile):
            part = row[t0:t0 + tile]
            if np.exp2(part - m).sum() > 2.0 ** 64:
                m = max(m, part.max())
                counts[i] += 1
    return counts


@pytest.mark.parametrize("d", [64, 256])
def test_reference_move_rescales_o(fa, d):
    """Scores that climb tile by tile, so the reference maximum moves, at
    different rates within one warp. Query row i carries a_i in
    {0, 1/8, 1/2, 1} (cycling, so every 32-row warp holds all four) in
    column 0, key j carries 400 * (j // 128) there (exact in bf16), the other
    columns small noise; with scale 1/8 a key tile raises a row's scores by
    72 a_i in log2 units. Rows with a_i = 1 move their reference maximum on
    every later tile (seven times); a_i = 1/2 every other tile; a_i = 1/8 at
    most once; a_i = 0 never. d = 64 runs the two-tile kernel (maximum taken
    before the exponentials, reference_moves), d = 256 the one-tile kernel
    (exponentiate, redo past 2^64, reference_redos). Without the move, tile
    7's probabilities for a_i = 1 would be exp2(505) = inf in fp32 and O would
    not be finite, so a finite O within the tolerance shows that the rescale
    of O and l ran."""
    N, scale = 1024, 0.125
    g = torch.Generator().manual_seed(3)
    q = 0.5 * torch.randn(1, 1, N, d, generator=g) * (64 / d) ** 0.5
    k = 0.5 * torch.randn(1, 1, N, d, generator=g)
    v = torch.randn(1, 1, N, d, generator=g)
    q[0, 0, :, 0] = torch.tensor([0.0, 0.125, 0.5, 1.0]).repeat(N // 4)
    k[0, 0, :, 0] = 400.0 * (torch.arange(N) // 128).float()
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    assert torch.equal(k[0, 0, :, 0].float(), 400.0 * (torch.arange(N) // 128).float())
    rule = reference_moves if d <= 128 else reference_redos
    for causal in (False, True):
        moves = rule(q, k, scale, causal)
        assert moves.max() == 7
        first = 256 if causal else 0     # causal rows of the first two tiles see at most 2 tiles
        for w0 in range(first, N, 32):   # every warp mixes rows that move their reference and rows that do not
            warp = moves[w0:w0 + 32]
            assert (warp >= 1).any() and (warp == 0).any(), (causal, w0, warp)
        err = check_full(fa, q, k, v, causal, scale=scale, what=f"climbing scores causal={causal} d={d}")
        print(f"climbing scores causal={causal} d={d}: reference moves per row max {moves.max()}, "
              f"total {moves.sum()}; max|dO| {err[0]:.3e} mean|dO| {err[1]:.3e}")


# ----------------------------------------------------------------- pins on the GPU path
def test_gpu_zero_query_gives_prefix_mean(fa):
    N, d = 384, 128
    q = torch.zeros(1, 2, N, d, dtype=torch.bfloat16)
    _, k, v, _ = workloads.make_custom(1, 2, N, d, seed=4)
    o, lse = run_gpu(fa, q, k, v, causal=True)
    vv = v.double().numpy()
    csum = np.cumsum(vv, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    assert np.abs(o - csum).max() <= MAX_ABS
    assert np.abs(lse - np.log(np.arange(1, N + 1))[None, None]).max() <= 1e-4


def test_gpu_constant_values(fa):
    q, k, _, _ = workloads.make_custom(2, 2, 257, 64, seed=5)
    v = torch.full_like(q, 1.5)
    o, _ = run_gpu(fa, q, k, v, causal=False)
    assert np.abs(o - 1.5).max() == 0.0  # weights sum to 1; 1.5 is exact in bf16


def test_deterministic(fa):
    q, k, v, _ = workloads.make_custom(2, 4, 1000, 128, seed=8)
    a = run_gpu(fa, q, k, v, True)
    b = run_gpu(fa, q, k, v, True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_guard_regions_untouched(fa):
    """O and lse live inside larger buffers; the bytes around them must
    survive the call (no out-of-bounds writes at ragged tails)."""
    B, H, N, d = 1, 3, 200, 128
    q, k, v, _ = workloads.make_custom(B, H, N, d, seed=12)
    dev = torch.device("cuda:0")
    pad_o, pad_l = 4096, 1024
    ob = torch.full((2 * pad_o + B * H * N * d,), 7.0, dtype=torch.bfloat16, device=dev)
    lb = torch.full((2 * pad_l + B * H * N,), 7.0, dtype=torch.float32, device=dev)
    out = ob[pad_o:pad_o + B * H * N * d].view(B, H, N, d)
    lse = lb[pad_l:pad_l + B * H * N].view(B, H, N)
    fa.attention(q.to(dev), k.to(dev), v.to(dev), causal=True, out=out, lse=lse)
    torch.cuda.synchronize()
    assert bool((ob[:pad_o] == 7.0).all()) and bool((ob[-pad_o:] == 7.0).all())
    assert bool((lb[:pad_l] == 7.0).all()) and bool((lb[-pad_l:] == 7.0).all())


def test_invalid_arguments_on_device(fa):
    x = torch.zeros(1, 1, 128, 96, dtype=torch.bfloat16, device="cuda:0")
    with pytest.raises(fa.FAError) as e:
        fa.attention(x, x, x)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_last_device_error(None) == fa.FA_OK


def test_very_long_sequence_sampled(fa):
    """N = 131072 (1024 query tiles per head, units far past the SM count):
    sampled rows of every head against the oracle."""
    B, H, N, d = 1, 4, 131072, 128
    q, k, v, _ = workloads.make_custom(B, H, N, d, seed=131)
    o, lse = run_gpu(fa, q, k, v, True)
    rows = workloads.sample_rows(N, seed=13, n_random=24, edge=4)
    o_ref, lse_ref = oracle.attention(q, k, v, 1 / math.sqrt(d), causal=True, rows=rows)
    compare(o[:, :, rows], lse[:, :, rows], o_ref, lse_ref, "N=131072 causal")

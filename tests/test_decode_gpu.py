"""GPU parity of the transposed decoding tile (bf16, d = 128, a K/V group's
query heads times the query rows within 8 columns), reached through
fa_fwd_splitkv, against the fp64 oracle, with the tolerances of the square
forward (tests/test_parity_gpu.py). Shapes with 9 or more columns take the
general kernel; both sides of that limit are checked."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.test_splitkv_gpu import check, run_splitkv

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


@pytest.mark.parametrize("H,H_kv,Nq", [
    (8, 1, 1),      # 8 heads of one group: every column a head
    (4, 1, 2),      # 4 heads x 2 rows
    (2, 2, 8),      # one head per group, 8 rows
    (3, 1, 2),      # 6 columns, 2 padding
    (1, 1, 9),      # 9 columns: the general kernel
    (16, 1, 1),     # 16 columns: the general kernel
])
@pytest.mark.parametrize("causal", [False, True])
def test_column_limits(fa, H, H_kv, Nq, causal):
    q, k, v, _ = workloads.make_qkv(2, H, H_kv, Nq, 1500, 128, seed=8000 + H * 31 + Nq)
    for splits in (1, 3):
        check(fa, q, k, v, causal, splits,
              what=f"H={H} H_kv={H_kv} Nq={Nq} causal={causal} splits={splits}")


def test_reference_moves_every_tile(fa):
    """Scores that grow by more than 64 log2 units from one key tile to the
    next (q and every key of tile t along one axis, the keys scaled by t), so
    every column's reference maximum moves, and O and the sums are rescaled,
    at every tile. The exact result is the mean of the last tile's V rows."""
    B, H, H_kv, Nq, Nk, d = 1, 4, 1, 2, 20 * 128, 128
    q = torch.zeros(B, H, Nq, d)
    q[..., 0] = 32.0
    k = torch.zeros(B, H_kv, Nk, d)
    k[..., 0] = 16.0 * (torch.arange(Nk) // 128).float()
    g = torch.Generator().manual_seed(3)
    v = torch.randn(B, H_kv, Nk, d, generator=g)
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    # 32 * 16 per tile step, times scale * log2(e) = 0.1275: 65.3 log2 units > 64
    assert 32 * 16 / math.sqrt(d) * math.log2(math.e) > 64
    for splits in (1, 4):
        check(fa, q, k, v, False, splits, what=f"moving reference splits={splits}")


def test_empty_and_tiny_caches(fa):
    """kv_len 0 (O = 0, lse = -inf), 1 and 129 keys, causal and not."""
    q, k, v, _ = workloads.make_qkv(3, 8, 2, 1, 640, 128, seed=8100)
    kv_len = torch.tensor([0, 1, 129], dtype=torch.int32)
    for causal in (False, True):
        for splits in (1, 2, 6):
            check(fa, q, k, v, causal, splits, kv_len,
                  what=f"tiny caches causal={causal} splits={splits}")
    out, lse = run_splitkv(fa, q, k, v, False, 2, kv_len)
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


N_CASES = 24


@pytest.mark.parametrize("case", range(N_CASES))
def test_random_decoding_shapes(fa, case):
    """Seeded random shapes within the tile's limits: group size, query rows,
    key count, causal, key padding, key ranges, Q magnitude."""
    rng = np.random.default_rng(99991 + 7919 * case)
    G = int(rng.choice([1, 2, 4, 8]))
    Nq = int(rng.integers(1, 8 // G + 1))
    H_kv = int(rng.integers(1, 4))
    H = H_kv * G
    B = int(rng.integers(1, 4))
    Nk = int(rng.integers(Nq, 3000))
    causal = bool(rng.integers(0, 2))
    splits = [None, 1, 2, 3, 7][int(rng.integers(0, 5))]
    q_mult = float(rng.choice([1.0, 2.0, 4.0]))
    kv_len = None
    if rng.random() < 0.4:
        kv_len = torch.from_numpy(rng.integers(0, Nk + 1, size=B).astype(np.int32))
    q, k, v, _ = workloads.make_qkv(B, H, H_kv, Nq, Nk, 128, seed=8200 + case)
    q = (q.float() * q_mult).to(torch.bfloat16)
    what = (f"case {case}: B{B} H{H} H_kv{H_kv} Nq{Nq} Nk{Nk} causal={causal} "
            f"splits={splits} q x {q_mult} kv_len={None if kv_len is None else kv_len.tolist()}")
    err = check(fa, q, k, v, causal, splits, kv_len, what=what)
    print(f"{what}: max|dO| {err[0]:.2e}")

"""GPU parity on seeded random configurations, every element against the fp64
oracle: head dim, batch, grouped K/V heads, ragged lengths, causal masking,
key padding, the scale, the magnitude of Q and, for the key-value-cache path
(fewer query rows than keys), the number of key ranges. Each case is drawn from
its own seed, so a failure names a configuration that can be rerun alone.
Sizes are kept small enough for the oracle to finish each case in well under a
second."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.test_parity_gpu import compare

pytestmark = pytest.mark.gpu

N_CASES = 48


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_18_b200 as fa
    from io_aware_exact_18_b200 import build
    build.build()
    fa.load_library()
    return fa


def draw(case):
    """One configuration: (path, B, H, H_kv, Nq, Nk, d, causal, kv_len, scale,
    q_mult, splits)."""
    rng = np.random.default_rng(20261203 + 7919 * case)
    path = "square" if case % 2 == 0 else "cache"
    d = int(rng.choice([64, 128, 256]))
    B = int(rng.integers(1, 4))
    H_kv = int(rng.integers(1, 4))
    G = int(rng.choice([1, 2, 4, 8]))
    H = H_kv * G
    if path == "square":
        Nk = int(rng.integers(1, 700))
        Nq = Nk
        splits = None
    else:
        Nk = int(rng.integers(1, 1500))
        Nq = int(rng.integers(1, min(Nk, 300) + 1))
        splits = [None, 1, 2, 3, 7][int(rng.integers(0, 5))]
    causal = bool(rng.integers(0, 2))
    kv_len = None
    if rng.random() < 0.5:
        kv_len = rng.integers(0, Nk + 1, size=B).astype(np.int32)
    scale = 1.0 / math.sqrt(d) if rng.random() < 0.6 else float(rng.uniform(0.05, 0.3))
    q_mult = float(rng.choice([1.0, 2.0, 4.0]))
    return path, B, H, H_kv, Nq, Nk, d, causal, kv_len, scale, q_mult, splits


@pytest.mark.parametrize("case", range(N_CASES))
def test_random_configuration(fa, case):
    path, B, H, H_kv, Nq, Nk, d, causal, kv_len, scale, q_mult, splits = draw(case)
    g = torch.Generator().manual_seed(1000 + case)
    q = (q_mult * torch.randn(B, H, Nq, d, generator=g)).to(torch.bfloat16)
    k = torch.randn(B, H_kv, Nk, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H_kv, Nk, d, generator=g).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    kvd = None if kv_len is None else torch.from_numpy(kv_len).to(dev)
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=dev)
    if path == "square":
        fa.attention(qd, kd, vd, scale=scale, causal=causal, kv_len=kvd, out=out, lse=lse)
    else:
        fa.decode_attention(qd, kd, vd, scale=scale, causal=causal, kv_len=kvd,
                            num_splits=splits, out=out, lse=lse)
    st = fa.fa_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    o_ref, lse_ref = oracle.attention(q, k, v, scale, causal=causal,
                                      kv_len=None if kv_len is None else kv_len)
    what = (f"case {case}: {path} B{B} H{H} H_kv{H_kv} Nq{Nq} Nk{Nk} d{d} causal={causal} "
            f"kv_len={None if kv_len is None else kv_len.tolist()} scale={scale:.4f} "
            f"q x {q_mult} splits={splits}")
    err = compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref, what)
    print(f"{what}: max|dO| {err[0]:.2e} mean|dO| {err[1]:.2e}")


N_BWD_CASES = 24


@pytest.mark.parametrize("case", range(N_BWD_CASES))
def test_random_backward(fa, case):
    """dQ, dK, dV of seeded random configurations (head dim 64 or 128, grouped
    K/V heads, ragged lengths, causal, key padding, Q magnitude) against the
    oracle's exact gradients, with the backward's bounds."""
    from tests.test_bwd_gpu import compare_grads, run_bwd
    rng = np.random.default_rng(777 + 104729 * case)
    d = int(rng.choice([64, 128]))
    B = int(rng.integers(1, 3))
    H_kv = int(rng.integers(1, 4))
    H = H_kv * int(rng.choice([1, 2, 4]))
    N = int(rng.integers(1, 600))
    causal = bool(rng.integers(0, 2))
    kv_range = (0, N) if rng.random() < 0.4 else None
    q_mult = float(rng.choice([1.0, 2.0]))
    import workloads
    q, k, v, do, kv_len = workloads.make_bwd_inputs(B, H, H_kv, N, d, seed=5000 + case,
                                                    kv_len_range=kv_range, q_mult=q_mult)
    what = (f"bwd case {case}: B{B} H{H} H_kv{H_kv} N{N} d{d} causal={causal} "
            f"kv_len={None if kv_len is None else kv_len.tolist()} q x {q_mult}")
    got = run_bwd(fa, q, k, v, do, causal, kv_len)
    ref = oracle.attention_bwd(q, k, v, do, 1.0 / math.sqrt(d), causal=causal, kv_len=kv_len)
    compare_grads(got, ref, what)
    print(what + ": ok")


N_FP8_CASES = 16


@pytest.mark.parametrize("case", range(N_FP8_CASES))
def test_random_fp8(fa, case):
    """The e4m3 forward on seeded random configurations (grouped K/V heads,
    ragged lengths, causal, key padding) against the oracle on the decoded
    inputs, with the e4m3 bounds."""
    from tests.test_fp8_gpu import check_fp8
    rng = np.random.default_rng(31337 + 15485863 * case)
    B = int(rng.integers(1, 3))
    H_kv = int(rng.integers(1, 4))
    H = H_kv * int(rng.choice([1, 2, 4]))
    N = int(rng.integers(1, 900))
    causal = bool(rng.integers(0, 2))
    kv_range = (0, N) if rng.random() < 0.4 else None
    err = check_fp8(fa, B, H, H_kv, N, causal, seed=7000 + case, kv_len_range=kv_range)
    print(f"fp8 case {case}: B{B} H{H} H_kv{H_kv} N{N} causal={causal} kv={kv_range}: "
          f"max|dO|/max|V| {err[0]:.2e}")


N_FP8_MORE = 16


@pytest.mark.parametrize("case", range(N_FP8_MORE))
def test_random_fp8_d256_and_cache(fa, case):
    """The e4m3 forward at d = 64 and 256 (square) and through the split-KV
    entry at d = 64, 128 and 256 (fewer query rows than keys, packed heads, key
    ranges) on seeded random configurations, with the e4m3 bounds."""
    from tests.test_fp8_gpu import check_fp8
    rng = np.random.default_rng(4242 + 7919 * case)
    B = int(rng.integers(1, 3))
    H_kv = int(rng.integers(1, 3))
    H = H_kv * int(rng.choice([1, 2, 4, 8]))
    causal = bool(rng.integers(0, 2))
    if case % 2 == 0:
        d, N = int(rng.choice([64, 256])), int(rng.integers(1, 700))
        Nk, splits = None, None
    else:
        d = int(rng.choice([64, 128, 256]))
        Nk = int(rng.integers(1, 1500))
        N = int(rng.integers(1, min(Nk, 200) + 1))
        splits = [None, 1, 2, 5][int(rng.integers(0, 4))]
    kv_hi = N if Nk is None else Nk
    kv_range = (0, kv_hi) if rng.random() < 0.4 else None
    err = check_fp8(fa, B, H, H_kv, N, causal, seed=7100 + case, kv_len_range=kv_range, d=d,
                    Nk=Nk, splits=splits)
    print(f"fp8 case {case}: B{B} H{H} H_kv{H_kv} N{N} Nk{Nk} d{d} causal={causal} "
          f"splits={splits} kv={kv_range}: max|dO|/max|V| {err[0]:.2e}")

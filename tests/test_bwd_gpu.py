"""GPU parity of the backward pass (fa_bwd) against the fp64 oracle's exact
gradients (oracle.attention_bwd).

O and lse come from this library's forward kernel on the same inputs, as in a
training step. Tolerances, per gradient tensor X in {dQ, dK, dV}, against the
oracle: max |dX| <= 2e-2 * max |X_ref| + 1e-5 and ||dX||_F <= 1e-2 * ||X_ref||_F
+ 1e-5 * sqrt(size). They follow from the arithmetic: P and dS are rounded to
bf16 (relative error 2^-9) before their tensor-core products, the gradients
are rounded to bf16 on output (2^-9), and D = dO . O uses the bf16 O. The
absolute floor covers fp32 cancellation in dP - D where the exact difference
is 0 (a row with one visible key has P = 1 and dS = 0 exactly, but dP and D
are summed in different fp32 orders).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

MAX_REL = 2e-2
FRO_REL = 1e-2
ABS_FLOOR = 1e-5


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_18_b200 as fa
    from io_aware_exact_18_b200 import build
    build.build()
    fa.load_library()
    return fa


def run_bwd(fa, q, k, v, do, causal, kv_len=None, poison=True):
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (x.to(dev).contiguous() for x in (q, k, v, do))
    kvd = None if kv_len is None else kv_len.to(dev)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention(qd, kd, vd, scale=scale, causal=causal, kv_len=kvd)
    grads = [torch.full_like(x, float("nan")) for x in (qd, kd, vd)]
    ws = torch.empty(fa.fa_bwd_workspace_bytes(*q.shape[:3]), dtype=torch.uint8, device=dev)
    if poison:   # the workspace needs no initialisation
        ws.view(torch.float32).fill_(float("nan"))
    fa.attention_bwd(qd, kd, vd, o, lse, dod, scale=scale, causal=causal, kv_len=kvd,
                     dq=grads[0], dk=grads[1], dv=grads[2], workspace=ws)
    st = fa.fa_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return grads


def compare_grads(got, ref, what):
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        g = g.double().cpu().numpy()
        assert not np.isnan(g).any(), f"{what}: {name} has unwritten (NaN) elements"
        err = np.abs(g - r)
        scale = np.abs(r).max()
        assert err.max() <= MAX_REL * scale + ABS_FLOOR, \
            f"{what}: {name} max|d| = {err.max():.3e} vs max|ref| = {scale:.3e}"
        fro, ref_fro = np.linalg.norm(err), np.linalg.norm(r)
        assert fro <= FRO_REL * ref_fro + ABS_FLOOR * math.sqrt(err.size), \
            f"{what}: {name} Frobenius error {fro:.3e} vs {ref_fro:.3e}"


def check(fa, q, k, v, do, causal, kv_len=None, what=""):
    got = run_bwd(fa, q, k, v, do, causal, kv_len)
    ref = oracle.attention_bwd(q, k, v, do, 1.0 / math.sqrt(q.shape[-1]), causal=causal,
                               kv_len=kv_len)
    compare_grads(got, ref, what)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 128, 129, 300])
def test_bwd_ragged_lengths(fa, N, causal, d):
    q, k, v, do, _ = workloads.make_bwd_inputs(1, 2, 2, N, d, seed=5000 + N + d + causal)
    check(fa, q, k, v, do, causal, what=f"N={N} causal={causal} d={d}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,H_kv", [(8, 2), (6, 1)])
def test_bwd_grouped_heads(fa, H, H_kv, causal):
    """dK, dV of a shared K/V head sum over its group of query heads."""
    q, k, v, do, kvl = workloads.make_bwd_inputs(2, H, H_kv, 256, 128, seed=5100 + H,
                                                 kv_len_range=(100, 256))
    check(fa, q, k, v, do, causal, None, what=f"H={H} H_kv={H_kv} causal={causal}")
    check(fa, q, k, v, do, causal, kvl, what=f"H={H} H_kv={H_kv} causal={causal} kv_len")


def test_bwd_key_padding_edges(fa):
    """kv_len 0 (no visible key: every gradient 0), short and full lengths."""
    q, k, v, do, _ = workloads.make_bwd_inputs(3, 2, 2, 300, 128, seed=5200)
    kvl = torch.tensor([0, 50, 300], dtype=torch.int32)
    for causal in (False, True):
        got = run_bwd(fa, q, k, v, do, causal, kvl)
        ref = oracle.attention_bwd(q, k, v, do, 1.0 / math.sqrt(128), causal=causal,
                                   kv_len=kvl)
        for g in got:
            assert torch.all(g[0] == 0), "batch with kv_len = 0 must get zero gradients"
        compare_grads(got, ref, f"kv_len edges causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_several_tiles(fa, causal):
    q, k, v, do, _ = workloads.make_bwd_inputs(2, 4, 4, 1024, 128, seed=5300 + causal)
    check(fa, q, k, v, do, causal, what=f"N=1024 causal={causal}")


def test_bwd_is_deterministic(fa):
    q, k, v, do, _ = workloads.make_bwd_inputs(1, 4, 2, 700, 128, seed=5400)
    a = run_bwd(fa, q, k, v, do, True)
    b = run_bwd(fa, q, k, v, do, True, poison=False)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_full_size_sampled(fa):
    """The backward the benchmark times (B1 H32 N16384 d128 causal, its inputs):
    dQ on sampled rows of every head against the oracle's row-by-row dQ; dK
    and dV element by element on three key tiles (the first, which every
    query row sees, one in the middle and the last, which few rows see) of
    the first and the last head against the oracle's key-row gradients; and
    the two invariants of the definition for dK and dV on every head
    (sum_j dK_j = 0; sum_j dV_j = sum_i dO_i, every causal row seeing a key),
    each within 1 % of the summed magnitudes."""
    w = workloads.get(5)
    q, k, v, do, _ = workloads.make_bwd_inputs(w.B, w.H, w.H, w.N, w.d, seed=w.index + 100)
    dq, dk, dv = run_bwd(fa, q, k, v, do, True)
    rows = workloads.sample_rows(w.N, seed=77, n_random=32, edge=8)
    ref = oracle.attention_bwd_dq_rows(q, k, v, do, w.scale, rows, causal=True)
    got = dq[:, :, rows].double().cpu().numpy()
    err = np.abs(got - ref)
    assert err.max() <= MAX_REL * np.abs(ref).max() + ABS_FLOOR, f"dQ rows max|d| {err.max():.3e}"
    assert np.linalg.norm(err) <= FRO_REL * np.linalg.norm(ref) + ABS_FLOOR * math.sqrt(err.size)
    heads = [0, w.H - 1]
    keys = list(range(0, 128)) + list(range(w.N // 2, w.N // 2 + 128)) + \
        list(range(w.N - 128, w.N))
    sel = [x[:, heads].contiguous() for x in (q, k, v, do)]
    dk_ref, dv_ref = oracle.attention_bwd_kv_rows(*sel, w.scale, keys, causal=True)
    for name, g, r in (("dK", dk, dk_ref), ("dV", dv, dv_ref)):
        got = g[:, heads][:, :, keys].double().cpu().numpy()
        err = np.abs(got - r)
        assert err.max() <= MAX_REL * np.abs(r).max() + ABS_FLOOR, \
            f"{name} key rows max|d| {err.max():.3e} vs max|ref| {np.abs(r).max():.3e}"
        assert np.linalg.norm(err) <= FRO_REL * np.linalg.norm(r) + \
            ABS_FLOOR * math.sqrt(err.size), f"{name} key rows Frobenius error"
    dk64, dv64 = dk.double(), dv.double()
    sum_dk = dk64.sum(dim=2).abs().sum(dim=-1)
    assert torch.all(sum_dk <= 1e-2 * dk64.abs().sum(dim=(2, 3))), "sum_j dK_j != 0"
    diff = (dv64.sum(dim=2) - do.double().to(dv.device).sum(dim=2)).abs().sum(dim=-1)
    assert torch.all(diff <= 1e-2 * dv64.abs().sum(dim=(2, 3))), "sum_j dV_j != sum_i dO_i"

"""fa_fwd_splitkv_static (split-KV with the library's own per-device scratch,
no allocation per call) against fa_fwd_splitkv with a caller workspace.

Kept in its own file, collected last, so that it also runs after every other
GPU test in one process; it passes alone in a fresh process as well. Both
entry points are called through the C ABI.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from tests.test_parity_gpu import MAX_ABS, MEAN_ABS

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


@pytest.mark.parametrize("B,H,H_kv,Nq,Nk,d,splits", [
    (4, 8, 2, 1, 3000, 128, 6),
    (2, 6, 6, 5, 1000, 64, 3),
    (1, 4, 1, 130, 2048, 256, 4),
])
def test_static_scratch_matches_workspace_entry(fa, B, H, H_kv, Nq, Nk, d, splits):
    q, k, v, _ = workloads.make_qkv(B, H, H_kv, Nq, Nk, d, seed=900 + Nq + d)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    scale = 1.0 / math.sqrt(d)
    s = torch.cuda.current_stream().cuda_stream
    need = fa.fa_splitkv_workspace_bytes(B, H, Nq, d, splits)
    assert 0 < need <= fa.FA_STATIC_SCRATCH_BYTES
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    o_ref = torch.empty_like(qd)
    l_ref = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    st = fa.fa_fwd_splitkv(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o_ref.data_ptr(),
                           l_ref.data_ptr(), B, H, H_kv, Nq, Nk, d, scale, 1, None, splits,
                           ws.data_ptr(), need, s)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    for call in range(2):   # two calls in a row reuse the same scratch
        o = torch.full_like(qd, float("nan"))
        lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=dev)
        st = fa.fa_fwd_splitkv_static(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                                      o.data_ptr(), lse.data_ptr(), B, H, H_kv, Nq, Nk, d,
                                      scale, 1, None, splits, s)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        st = fa.fa_last_device_error(s)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        a = o.double().cpu().numpy()
        b = o_ref.double().cpu().numpy()
        assert not np.isnan(a).any(), f"call {call}: unwritten output"
        err = np.abs(a - b)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, f"call {call}: {err.max()}"
        la, lb = lse.double().cpu().numpy(), l_ref.double().cpu().numpy()
        assert np.allclose(la, lb, rtol=1e-6, atol=1e-6), f"call {call}: lse"


def test_static_scratch_rejects_requests_beyond_its_size(fa):
    B, H, H_kv, Nq, Nk, d, splits = 64, 32, 8, 16, 4096, 128, 16
    assert fa.fa_splitkv_workspace_bytes(B, H, Nq, d, splits) > fa.FA_STATIC_SCRATCH_BYTES
    P = 1 << 40   # never dereferenced: the size is checked before any CUDA call
    st = fa.fa_fwd_splitkv_static(P, P + (1 << 32), P + (2 << 32), P + (3 << 32), P + (4 << 32),
                                  B, H, H_kv, Nq, Nk, d, 0.088, 1, None, splits, None)
    assert st == fa.FA_ERR_INVALID_ARG

"""fa_fwd_splitkv_static (split-KV with the library's own per-device scratch,
no allocation per call) against fa_fwd_splitkv with a caller workspace.

Both entry points run the same kernels on the same inputs, so their outputs
must agree bit for bit; each shape is also checked against the fp64 oracle.
Kept in its own file, collected last, so that it also runs after every other
GPU test in one process; it passes alone in a fresh process as well. Both
entry points are called through the C ABI.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.test_parity_gpu import compare

pytestmark = pytest.mark.gpu

# The scratch needs splits * rows * (d + 1) * 4 bytes (rows = B * H * Nq), with
# the O part rounded up to 256 bytes; (d + 1) * 4 never divides 2^24, so no
# shape fills the 16 MiB exactly. AT_LIMIT is the largest whole shape of its
# form: 4 * 15 * 272 rows-and-ranges at d = 256 need 16776960 bytes, 256 short.
AT_LIMIT = (1, 15, 5, 272, 2048, 256, 4)


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_18_b200 as fa
    from io_aware_exact_18_b200 import build
    build.build()
    fa.load_library()
    return fa


@pytest.mark.parametrize("B,H,H_kv,Nq,Nk,d,splits,kv", [
    (4, 8, 2, 1, 3000, 128, 6, None),
    (2, 6, 6, 5, 1000, 64, 3, None),
    (1, 4, 1, 130, 2048, 256, 4, None),
    (3, 8, 2, 2, 2500, 128, 5, [2500, 700, 1]),
    AT_LIMIT + (None,),
])
def test_static_scratch_matches_workspace_entry(fa, B, H, H_kv, Nq, Nk, d, splits, kv):
    q, k, v, _ = workloads.make_qkv(B, H, H_kv, Nq, Nk, d, seed=900 + Nq + d)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    kv_len = None if kv is None else torch.tensor(kv, dtype=torch.int32)
    kvd = None if kv_len is None else kv_len.to(dev)
    kvp = None if kvd is None else kvd.data_ptr()
    scale = 1.0 / math.sqrt(d)
    s = torch.cuda.current_stream().cuda_stream
    need = fa.fa_splitkv_workspace_bytes(B, H, Nq, d, splits)
    assert 0 < need <= fa.FA_STATIC_SCRATCH_BYTES
    if (B, H, H_kv, Nq, Nk, d, splits) == AT_LIMIT:
        assert fa.FA_STATIC_SCRATCH_BYTES - need == 256
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    o_ref = torch.empty_like(qd)
    l_ref = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    st = fa.fa_fwd_splitkv(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o_ref.data_ptr(),
                           l_ref.data_ptr(), B, H, H_kv, Nq, Nk, d, scale, 1, kvp, splits,
                           ws.data_ptr(), need, s)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    o64, l64 = oracle.attention(q, k, v, scale, causal=True, kv_len=kv_len)
    for call in range(2):   # two calls in a row reuse the same scratch
        o = torch.full_like(qd, float("nan"))
        lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=dev)
        st = fa.fa_fwd_splitkv_static(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                                      o.data_ptr(), lse.data_ptr(), B, H, H_kv, Nq, Nk, d,
                                      scale, 1, kvp, splits, s)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        st = fa.fa_last_device_error(s)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        assert torch.equal(o, o_ref), f"call {call}: O differs from the workspace entry point"
        assert torch.equal(lse, l_ref), f"call {call}: lse differs from the workspace entry point"
        compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), o64, l64,
                f"static scratch call {call}")


def test_static_scratch_rejects_requests_beyond_its_size(fa):
    B, H, H_kv, Nq, Nk, d, splits = AT_LIMIT
    over = (B, H, H_kv, Nq + 1, Nk, d, splits)   # one query row more than fits
    assert fa.fa_splitkv_workspace_bytes(B, H, Nq + 1, d, splits) > fa.FA_STATIC_SCRATCH_BYTES
    P = 1 << 40   # never dereferenced: the size is checked before any CUDA call
    st = fa.fa_fwd_splitkv_static(P, P + (1 << 32), P + (2 << 32), P + (3 << 32), P + (4 << 32),
                                  *over[:6], 0.0625, 1, None, over[6], None)
    assert st == fa.FA_ERR_INVALID_ARG
    big = (64, 32, 8, 16, 4096, 128, 16)
    assert fa.fa_splitkv_workspace_bytes(64, 32, 16, 128, 16) > fa.FA_STATIC_SCRATCH_BYTES
    st = fa.fa_fwd_splitkv_static(P, P + (1 << 32), P + (2 << 32), P + (3 << 32), P + (4 << 32),
                                  *big[:6], 0.088, 1, None, big[6], None)
    assert st == fa.FA_ERR_INVALID_ARG


def test_static_scratch_same_status_codes_as_workspace_entry(fa):
    """Argument errors other than the size come back as fa_fwd_splitkv gives
    them (an unsupported head dim is FA_ERR_UNSUPPORTED, not an argument
    error), before any CUDA call."""
    P = 1 << 40
    for d, want in ((96, fa.FA_ERR_UNSUPPORTED), (128, fa.FA_ERR_INVALID_ARG)):
        H_kv = 3 if d == 128 else 2          # 8 % 3 != 0: invalid grouping
        st = fa.fa_fwd_splitkv_static(P, P + (1 << 32), P + (2 << 32), P + (3 << 32),
                                      P + (4 << 32), 1, 8, H_kv, 1, 512, d, 0.1, 1, None, 4,
                                      None)
        assert st == want, (d, st)

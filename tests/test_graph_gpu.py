"""The library's calls captured in a CUDA graph and replayed: a square forward,
a split-KV decode with several key ranges (whose merge is launched as a
programmatic dependent of the decoding kernel) and a backward. A replay on new
inputs, written in place into the captured buffers, must give the same bits as
eager calls on those inputs, and the decode must match the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

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


def test_capture_and_replay(fa):
    dev = torch.device("cuda:0")
    q, k, v, do, _ = workloads.make_bwd_inputs(1, 4, 2, 640, 128, seed=91)
    qs, ks, vs, _ = workloads.make_qkv(2, 8, 2, 1, 3000, 128, seed=92)
    bufs = [x.to(dev) for x in (q, k, v, do, qs, ks, vs)]
    qd, kd, vd, dod, qsd, ksd, vsd = bufs

    def step():
        o, lse = fa.attention(qd, kd, vd, causal=True)
        od, ld = fa.decode_attention(qsd, ksd, vsd, causal=True, num_splits=4)
        dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, lse, dod, causal=True)
        return o, lse, od, ld, dq, dk, dv

    # warm-up on a side stream (first calls probe the device and set kernel
    # attributes, which a capture must not see)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        captured = step()

    # new inputs written into the captured buffers, then a replay
    q2, k2, v2, do2, _ = workloads.make_bwd_inputs(1, 4, 2, 640, 128, seed=93)
    qs2, ks2, vs2, _ = workloads.make_qkv(2, 8, 2, 1, 3000, 128, seed=94)
    for dst, src in zip(bufs, (q2, k2, v2, do2, qs2, ks2, vs2)):
        dst.copy_(src.to(dev))
    graph.replay()
    torch.cuda.synchronize()
    st = fa.fa_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    replayed = [x.clone() for x in captured]

    eager = step()
    torch.cuda.synchronize()
    names = ("O", "lse", "decode O", "decode lse", "dQ", "dK", "dV")
    for name, a, b in zip(names, replayed, eager):
        assert torch.equal(a, b), f"{name}: replay differs from the eager call"

    o_ref, lse_ref = oracle.attention(qs2, ks2, vs2, 1.0 / math.sqrt(128), causal=True)
    err = np.abs(replayed[2].double().cpu().numpy() - o_ref)
    assert err.max() <= 2e-2, f"decode max|dO| {err.max():.3e}"
    lerr = np.abs(replayed[3].double().cpu().numpy() - lse_ref) / np.maximum(np.abs(lse_ref), 1.0)
    assert lerr.max() <= 1e-3

"""GPU: a bounded wait that is made to run out ends its kernel with an error
status the host can read, and the context stays usable afterwards. Nothing
here faults, traps or hangs the GPU: the wait is on a shared-memory barrier
nobody completes and gives up after 20 ms.

While the device status word is set, every launch skips its work; its outputs
then read NaN, so a caller who does not read the word finds no stale values."""
import math
import time

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


def test_bounded_wait_runs_out_and_is_reported(fa):
    stream = torch.cuda.current_stream().cuda_stream
    assert fa.fa_last_device_error(stream) == fa.FA_OK      # clean start
    t0 = time.time()
    assert fa.fa_watchdog_selftest(20_000_000, stream) == fa.FA_OK
    assert fa.fa_last_device_error(stream) == fa.FA_ERR_TIMEOUT
    assert time.time() - t0 < 10.0
    assert fa.fa_last_device_error(stream) == fa.FA_OK      # the word was cleared
    # the context still works: a normal forward matches the oracle
    w = workloads.get(1)
    q, k, v, _ = workloads.make_inputs(w)
    o, lse = fa.attention(q.cuda(), k.cuda(), v.cuda(), scale=w.scale)
    assert fa.fa_last_device_error(stream) == fa.FA_OK
    o_ref, _ = oracle.attention(q, k, v, w.scale)
    assert np.abs(o.double().cpu().numpy() - o_ref).max() <= 2e-2


def test_skipped_launches_write_nan(fa):
    """After the selftest sets the word (and nobody reads it): the square
    forward at d = 64, 128 and 256, the e4m3 forward, a split-KV call through
    the library's static scratch (its merge must not mix stale partials) and
    the backward each fill their outputs with NaN. Then the word reads
    FA_ERR_TIMEOUT, and the next forward matches the oracle again."""
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream().cuda_stream
    assert fa.fa_last_device_error(stream) == fa.FA_OK
    # fill the static scratch with a finished, valid merge first, so a stale
    # merge would produce finite values
    qs, ks, vs, _ = workloads.make_qkv(2, 8, 2, 3, 900, 128, seed=41)
    qs, ks, vs = qs.to(dev), ks.to(dev), vs.to(dev)
    o_s = torch.empty_like(qs)
    l_s = torch.empty((2, 8, 3), dtype=torch.float32, device=dev)
    args = (qs.data_ptr(), ks.data_ptr(), vs.data_ptr(), o_s.data_ptr(), l_s.data_ptr(),
            2, 8, 2, 3, 900, 128, 1 / math.sqrt(128), 1, None, 4, stream)
    assert fa.fa_fwd_splitkv_static(*args) == fa.FA_OK
    assert fa.fa_last_device_error(stream) == fa.FA_OK
    assert torch.isfinite(o_s).all()

    assert fa.fa_watchdog_selftest(20_000_000, stream) == fa.FA_OK
    torch.cuda.synchronize()
    outs = []
    for d in (64, 128, 256):
        q, k, v, _ = workloads.make_custom(2, 3, 300, d, seed=40 + d)
        o = torch.zeros((2, 3, 300, d), dtype=torch.bfloat16, device=dev)
        lse = torch.zeros((2, 3, 300), dtype=torch.float32, device=dev)
        fa.attention(q.to(dev), k.to(dev), v.to(dev), causal=True, out=o, lse=lse)
        outs += [(f"fwd d={d}", o), (f"fwd d={d} lse", lse)]
    q8, k8, v8, sc, _ = workloads.make_fp8_inputs(1, 2, 2, 256, 128, seed=44)
    o8, l8 = fa.attention_fp8(q8.to(dev), k8.to(dev), v8.to(dev), *sc, causal=True)
    outs += [("e4m3", o8), ("e4m3 lse", l8)]
    o_s.zero_()
    l_s.zero_()
    assert fa.fa_fwd_splitkv_static(*args) == fa.FA_OK
    outs += [("split-KV static", o_s), ("split-KV static lse", l_s)]
    qb, kb, vb, dob, _ = workloads.make_bwd_inputs(1, 2, 2, 200, 128, seed=45)
    qb, kb, vb, dob = (x.to(dev) for x in (qb, kb, vb, dob))
    ob = torch.zeros_like(qb)
    lb = torch.zeros((1, 2, 200), dtype=torch.float32, device=dev)
    grads = [torch.zeros_like(x) for x in (qb, kb, vb)]
    fa.attention_bwd(qb, kb, vb, ob, lb, dob, causal=True, dq=grads[0], dk=grads[1],
                     dv=grads[2])
    outs += [("bwd dQ", grads[0]), ("bwd dK", grads[1]), ("bwd dV", grads[2])]
    torch.cuda.synchronize()
    for name, t in outs:
        assert torch.isnan(t.float()).all(), f"{name}: a skipped launch left non-NaN values"
    assert fa.fa_last_device_error(stream) == fa.FA_ERR_TIMEOUT
    assert fa.fa_last_device_error(stream) == fa.FA_OK
    w = workloads.get(1)
    q, k, v, _ = workloads.make_inputs(w)
    o, _ = fa.attention(q.to(dev), k.to(dev), v.to(dev), scale=w.scale)
    o_ref, _ = oracle.attention(q, k, v, w.scale)
    assert np.abs(o.double().cpu().numpy() - o_ref).max() <= 2e-2

"""GPU: a bounded wait that is made to run out ends its kernel with an error
status the host can read, and the context stays usable afterwards. Nothing
here faults, traps or hangs the GPU: the wait is on a shared-memory barrier
nobody completes and gives up after 20 ms."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_18_b200 as fa
    from io_aware_exact_18_b200 import build
    build.build()
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

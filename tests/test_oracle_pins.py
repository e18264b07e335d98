"""CPU-only: the oracle against its pins, its two entry routes, and edge cases."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    pin(lib)


def test_bf16_route_matches_fp64_route(lib):
    """bf16 bit patterns widened inside the oracle == fp64 inputs widened by torch."""
    q, k, v, _ = workloads.make_custom(2, 2, 77, 16, seed=5)
    o1, l1 = oracle.attention(q, k, v, 0.25, causal=True, lib=lib)
    o2, l2 = oracle.attention(q.double(), k.double(), v.double(), 0.25, causal=True, lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_row_subset_matches_full(lib):
    q, k, v, _ = workloads.make_custom(1, 3, 140, 8, seed=6)
    rows = [0, 1, 63, 64, 127, 128, 139]
    o, l = oracle.attention(q, k, v, 0.3, causal=True, lib=lib)
    os_, ls = oracle.attention(q, k, v, 0.3, causal=True, rows=rows, lib=lib)
    assert np.array_equal(o[:, :, rows], os_) and np.array_equal(l[:, :, rows], ls)


def test_thread_count_does_not_change_result(lib):
    q, k, v, _ = workloads.make_custom(1, 2, 200, 32, seed=7)
    o1, l1 = oracle.attention(q, k, v, 0.2, nthreads=1, lib=lib)
    o4, l4 = oracle.attention(q, k, v, 0.2, nthreads=4, lib=lib)
    assert np.array_equal(o1, o4) and np.array_equal(l1, l4)


def test_rejects_bad_arguments(lib):
    q = np.zeros((1, 1, 4, 2))
    with pytest.raises(RuntimeError):
        oracle.attention(q, q, q, float("nan"), lib=lib)
    with pytest.raises(ValueError):
        oracle.attention(q, q, np.zeros((1, 1, 5, 2)), 1.0, lib=lib)


def test_workload_generator_is_deterministic():
    w = workloads.get(2)
    a = workloads.make_inputs(w)
    b = workloads.make_inputs(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    q, k, v, kv_len = a
    assert q.dtype == torch.bfloat16 and q.shape == (16, 16, 512, 64)
    assert kv_len.dtype == torch.int32 and kv_len.shape == (16,)
    assert int(kv_len.min()) >= 256 and int(kv_len.max()) <= 512
    # Q x 4 case: exact power-of-two scaling of the bf16 draw
    w4 = workloads.Workload("t", 4, 1, 1, 16, 8, True, q_mult=4.0)
    q4, _, _, _ = workloads.make_inputs(w4, seed=3)
    w1 = workloads.Workload("t", 4, 1, 1, 16, 8, True)
    q1, _, _, _ = workloads.make_inputs(w1, seed=3)
    assert torch.equal(q4.float(), q1.float() * 4)


def test_flop_count_convention():
    assert workloads.get(5).flops() == pytest.approx(2.199023255552e12)
    assert workloads.get(1).flops() == 4 * 1 * 2 * 256 * 256 * 64

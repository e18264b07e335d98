"""CPU-only checks of bench.py's bookkeeping and of the no-fallback rule."""
import itertools
import os

import pytest
import torch

import bench
import workloads


@pytest.mark.parametrize("causal", [False, True])
def test_visible_pairs_matches_brute_force(causal):
    w = workloads.Workload("t", 0, 3, 2, 37, 64, causal)
    for kv_len in (None, torch.tensor([0, 20, 99], dtype=torch.int32)):
        lims = [37] * 3 if kv_len is None else [min(max(int(x), 0), 37) for x in kv_len]
        brute = sum(1 for b, i, j in itertools.product(range(3), range(37), range(37))
                    if j < lims[b] and (not causal or j <= i)) * w.H
        assert bench.visible_pairs(w, kv_len) == brute


def test_visible_pairs_of_the_workloads():
    w5 = workloads.get(5)
    assert bench.visible_pairs(w5) == w5.H * w5.N * (w5.N + 1) // 2
    assert 4.0 * w5.d * bench.visible_pairs(w5) == pytest.approx(w5.flops(), rel=1e-4)


def test_source_hash_ignores_comments(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_text("int a = 1; // one\n/* block */ int b = 2;\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [str(src)])
    monkeypatch.setattr(bench, "ROOT", "/")
    h1 = bench.kernel_source_hash()
    src.write_text("int a = 1;   // a different comment\n\n/* another */\nint b = 2;\n")
    assert bench.kernel_source_hash() == h1
    src.write_text("int a = 1; int b = 3;\n")
    assert bench.kernel_source_hash() != h1


def test_recorded_traffic_requires_matching_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic_x.txt").write_text("kernel_source_sha256_16: abc\ndram_bytes_per_launch: 123\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.recorded_traffic("x") == 123.0
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "def")
    assert bench.recorded_traffic("x") is None


def test_missing_extension_fails_loudly(tmp_path):
    import io_aware_exact_18_b200 as fa
    with pytest.raises(ImportError):
        fa.load_library(os.path.join(str(tmp_path), "libfa.so"))
